// gemv.cu -- the LUT binary GEMV y = W_hat x of the FluxBin page
// (Methodology, 2. Kernel innovation), written for sm_100a.
//
// W_hat = sum_k (alpha_r^(k) alpha_c^(k)^T) (.) B^(k)  +  salient refinement
// (1. Algorithm innovation; Hessian-guided saliency-aware hybrid bases).
//
// Work units.  A "virtual panel" is one panel (<= 256 columns) of one base,
// global or salient; the matrix has V of them.  Rows come in chunks of 32,
// one row per lane; an "item" is one chunk of one virtual panel (32 rows x
// <= 32 bytes).  A thread-block cluster of C CTAs owns one block of cpb
// chunks; CTA j of the cluster takes a contiguous, balanced slice of the V
// virtual panels, so the cluster covers every column of its rows.
//
// Per CTA (16 warps, or 8 for dependent calls; warp w owns chunks w and
// w + warps of the row block):
//   1. before the programmatic-launch wait: the weights of the first panels
//      start streaming into shared-memory slots (one bulk asynchronous copy
//      per panel of the row block, completion on an mbarrier), and the row
//      scales and per-panel descriptors are staged in shared memory;
//   2. per panel, all 256 threads build its byte tables in shared memory
//      (LUT-BSF: z = alpha_c * x, salient panels reading x[s_idx[t]] -- the
//      virtual columnar mapping -- and for each group of 8 columns the 256
//      sums sum_t (bit t of b ? +z_t : -z_t), each the sum of the two 4-column
//      tables of its nibbles), double-buffered, one CTA barrier per panel;
//   3. each lane walks its row's 32 bytes: one `prmt` merges a weight byte and
//      the lane's column offset into a table address, one shared load fetches
//      the partial sum, packed fp32x2 adds accumulate (a gather-add, no tensor
//      cores); each item's sum is scaled by alpha_r once (alpha_r applied in
//      the reduction) and added to the row's partial;
//   4. each CTA pushes its row partials into the shared memory of the CTA
//      that owns those rows, the cluster synchronises once, and each owner
//      sums its C inbox slots in rank order and writes y.  No workspace, no
//      atomics; deterministic.
//
// Byte tables: entry b of byte group q (columns 8q .. 8q+7 of the panel) is
// at b*256 + 4q bytes; the two buffers interleave, the second at +128.  Lane
// l at stored position u reads byte group (l+u) mod Bp (the rotation of the
// packed layout), so a warp's 32 lookups hit 32 different banks.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstddef>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <new>
#include <type_traits>
#include <vector>

#include "fb_internal.cuh"

namespace cg = cooperative_groups;

namespace fb {
namespace {

constexpr int kMaxCluster = 16;   // 16: non-portable cluster size (B200 allows it)
constexpr int kMaxSlotCluster = 8;   // gemv_kernel's plans stay within the portable size
constexpr int kMaxGroup = 4;            // matrices in one grouped call
// Two CTA shapes.  16 warps, one CTA per SM, up to 32 chunks per row block
// and three weight slots: calls flagged independent (fewest table builds per
// row).  8 warps, two CTAs per SM, up to 16 chunks and two slots: dependent
// calls (twice the CTAs in one wave, shorter panel lists per CTA).  Both give
// each warp two chunks of every panel.
template <int NW>
struct Shape {
    static constexpr int kSlots = NW == 16 ? 3 : 2;
    static constexpr int kMinBlocks = 16 / NW;     // CTAs per SM the registers allow
};
constexpr size_t kMaxDynSmem = 225 * 1024;   // dynamic shared memory per CTA
constexpr size_t kSmemPerSM = 228 * 1024;
constexpr size_t kStaticSmem = 1024;          // the kernel's static shared memory, rounded up
constexpr unsigned kKnownFlags = FB_GEMV_PDL | FB_GEMV_INDEPENDENT | FB_GEMV_TEST_WAIT_TIMEOUT;

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
    int nchunks, cpb;         // chunks (32 rows) in the matrix, per row block
    int ldx, ldy;
    unsigned flags;
    int C;
    int batch, tp;   // tokens of the call; tokens per pass (batched kernel: grid.z = passes)
    // Row scales: KR = K * ngr global row-scale vectors (ngr = 1, or N / G
    // for group-wise row scales, alpha_r[(k * ngr + g) * M + i]); hsplit = 1
    // when G = 128, which splits every panel into two half-panels.
    int G, ngr, KR, hsplit;
    int vsplit[kMaxCluster + 1];   // CTA j of a cluster: virtual panels [vsplit[j], vsplit[j+1])
    // Grouped calls: up to kMaxGroup matrices of one format (N, K, g, nS, Ks)
    // that read the same x.  Row blocks [rb_start[m], rb_start[m+1]) of the
    // grid belong to matrix m, whose fields replace the ones above at entry.
    int group;     // matrices in the call; 1: the fields above are the matrix
    int rb_base;   // set at entry: the first row block of this CTA's matrix
    int rb_start[kMaxGroup + 1];
    struct Mat {
        const uint8_t *planes;
        const float *alpha_r, *alpha_c;
        const uint8_t *s_planes;
        const float *s_alpha_r, *s_alpha_c;
        const uint32_t *s_idx;
        float *y;
        int M, M_pad, nchunks, pad;
    } mats[kMaxGroup];
};

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- bulk asynchronous copies into shared memory, signalled on mbarriers ----
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// One copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// global memory into this CTA's shared memory; the barrier's phase completes
// when the bytes have landed.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%2], %1;\n\t"
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%3], %1, [%2];\n\t}"
        ::"r"(dst), "r"(bytes), "r"(bar), "l"(src)
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// The same with cluster scope: the phase is completed by other CTAs' remote
// stores, which the waiting threads then read.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait for a barrier phase: gives up after kWaitLimitNs (or
// kWaitLimitIters polls) and returns false.
constexpr unsigned long long kWaitLimitNs = 200ull * 1000 * 1000;
constexpr int kWaitLimitIters = 1 << 24;
template <bool kCluster = false>
__device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    unsigned long long t0 = 0;
    for (int it = 0; it < kWaitLimitIters; ++it) {
        if (kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if ((it & 31) == 31) {
            const unsigned long long now = global_ns();
            if (t0 == 0)
                t0 = now;
            else if (now - t0 > kWaitLimitNs)
                return false;
        }
    }
    return false;
}

// Announce `bytes` of asynchronous transactions on a barrier (with this
// thread's arrival).
__device__ __forceinline__ void mbar_arrive_expect(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar), "r"(bytes)
        : "memory");
}
// One float into the shared memory of cluster CTA `rank` (at the address
// `local` has in this CTA), completing 4 bytes on that CTA's barrier at the
// address `bar` has here.
__device__ __forceinline__ void push_remote(uint32_t local, uint32_t bar, int rank, float v) {
    uint32_t ra, rb;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local), "r"(rank));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(bar), "r"(rank));
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(ra),
                 "r"(__float_as_uint(v)), "r"(rb)
                 : "memory");
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

// The 16 entries sum_{t<4} (bit t of a ? +1 : -1) * z_t, a = 0..15, as
// (+-z0 +- z1) + (+-z2 +- z3).
__device__ __forceinline__ void sums16(float z0, float z1, float z2, float z3, float (&e)[16]) {
    const float p01[4] = {__fadd_rn(-z0, -z1), __fadd_rn(z0, -z1), __fadd_rn(-z0, z1), __fadd_rn(z0, z1)};
    const float p23[4] = {__fadd_rn(-z2, -z3), __fadd_rn(z2, -z3), __fadd_rn(-z2, z3), __fadd_rn(z2, z3)};
#pragma unroll
    for (int a = 0; a < 16; ++a) e[a] = __fadd_rn(p01[a & 3], p23[a >> 2]);
}

// One virtual panel: its width, its scales and its columns.
struct VPanel {
    const float *ac;     // column scales of this base, or null (all ones)
    int col0;            // first column of the panel (global, or compact salient)
    int Bp;              // byte groups (width / 8)
    int kb;              // row-scale vector: k (k * ngr + g with group-wise scales), KR + k for salient ones
    int sal;             // 1 for salient panels
    int half;            // 0: every column; 1 / 2: only the first / second 128 columns
};

// Position of a virtual panel in the order global panels of base 0, 1, ...
// then salient ones; a CTA walks its slice one panel at a time.  With
// half-panels (hsplit), global panel position p' is panel p'/2, half p'%2.
struct PanelPos {
    int sal, k, p, h;
};

// Global virtual panels per base.
__host__ __device__ __forceinline__ int global_vpanels(int N, int hsplit) {
    return hsplit ? N / 128 : num_panels(N);
}

__device__ __forceinline__ PanelPos panel_pos(const GemvArgs &a, int v) {
    const int Pv = global_vpanels(a.N, a.hsplit), ng = Pv * a.K;
    PanelPos q;
    q.sal = v >= ng;
    const int r = q.sal ? v - ng : v, P = q.sal ? max(a.Ps, 1) : Pv;
    q.k = r / P;
    const int pp = r - q.k * P;
    q.p = (!q.sal && a.hsplit) ? pp >> 1 : pp;
    q.h = (!q.sal && a.hsplit) ? 1 + (pp & 1) : 0;
    return q;
}

__device__ __forceinline__ VPanel panel_at(const GemvArgs &a, const PanelPos &q) {
    const int ncols = q.sal ? a.nS_pad : a.N;
    VPanel r;
    r.sal = q.sal;
    r.half = q.h;
    r.col0 = q.p * kPanelCols;
    r.kb = q.sal ? a.KR + q.k
                 : q.k * a.ngr + (a.ngr > 1 ? (r.col0 + (q.h == 2 ? 128 : 0)) / a.G : 0);
    r.Bp = panel_width(ncols, q.p) >> 3;
    r.ac = q.sal ? a.s_alpha_c + (size_t)q.k * a.nS : (a.alpha_c ? a.alpha_c + (size_t)q.k * a.N : nullptr);
    return r;
}

// Chunk block 0 of a virtual panel in its planes buffer.
__device__ __forceinline__ const uint8_t *panel_planes(const GemvArgs &a, const PanelPos &q) {
    const int ncols = q.sal ? a.nS_pad : a.N;
    return (q.sal ? a.s_planes : a.planes) + (size_t)q.k * a.M_pad * (size_t)(ncols / 8) +
           (size_t)32 * q.p * a.M_pad;
}

// What a CTA needs of one of its panels, built once per CTA in shared
// memory: width, flags, row-scale vector, first column, scales, words.
struct PanelDesc {
    const float *ac;      // column scales of the panel's base, or null (all ones)
    const uint8_t *pl;    // chunk block 0 of the panel
    int info;             // Bp | sal << 8 | half << 9
    int col0;
    int kb;               // row-scale vector
    int pad;
};

__device__ __forceinline__ int desc_bp(const PanelDesc &d) { return d.info & 255; }
__device__ __forceinline__ int desc_sal(const PanelDesc &d) { return (d.info >> 8) & 1; }
__device__ __forceinline__ int desc_half(const PanelDesc &d) { return d.info >> 9; }

// The row-scale vector kb of the call (global, then salient).
__device__ __forceinline__ const float *row_scales(const GemvArgs &a, int kb) {
    return kb < a.KR ? a.alpha_r + (size_t)kb * a.M : a.s_alpha_r + (size_t)(kb - a.KR) * a.M;
}

__device__ __forceinline__ PanelDesc panel_desc(const GemvArgs &a, int v) {
    const PanelPos q = panel_pos(a, v);
    const VPanel vp = panel_at(a, q);
    PanelDesc d;
    d.ac = vp.ac;
    d.pl = panel_planes(a, q);
    d.info = vp.Bp | vp.sal << 8 | vp.half << 9;
    d.col0 = vp.col0;
    d.kb = vp.kb;
    d.pad = 0;
    return d;
}

// Column c of a panel: its scale alpha_c and the column of x it reads (-1:
// none: the other half of a half-panel, and the columns past a narrow
// panel's width, which build all-zero table columns).  With kDup, the
// columns past a narrow panel's width (Bp < 32 byte groups) instead repeat
// its columns, floor(32 / Bp) copies in all, so lanes of a warp that share a
// byte group can read different copies (narrow_offsets_dup).
template <bool kDup = false>
__device__ __forceinline__ void column_source(const GemvArgs &a, const PanelDesc &d, int c, float &ac, int &xi) {
    ac = 0.0f;
    xi = -1;
    const int w = desc_bp(d) * 8;
    if (c >= w) {
        if (!kDup || c >= (kPanelCols / w) * w) return;
        c -= (c / w) * w;
    }
    const int half = desc_half(d);
    if (half && (c >> 7) != half - 1) return;   // a half-panel: the other half's columns build zeros
    const int col = d.col0 + c;
    if (!desc_sal(d)) {
        xi = col;
        if (d.ac)
            ac = __ldg(d.ac + col);
        else
            ac = 1.0f;
    } else if (col < a.nS) {
        ac = __ldg(d.ac + col);
        const uint32_t jx = __ldg(a.s_idx + col);
        xi = jx < (uint32_t)a.N ? (int)jx : -1;   // an invalid index contributes 0
    }
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

// Column offsets of a narrow panel (Bp < 32): byte j of word m = 4 * ((lane
// + u) mod Bp) for u = 4m + j < Bp, and column 31 (built all zero) for the
// positions past Bp.  Narrow panels are rare, so this stays out of line.
struct Offsets {
    uint32_t w[8];
};
__device__ __noinline__ Offsets narrow_offsets(int lane, int Bp) {
    Offsets o;
    const int r = lane % Bp;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        uint32_t word = 0;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int u = 4 * m + jj;
            int q = r + u;
            q = q >= Bp ? q - Bp : q;
            q = u < Bp ? q : 31;
            word |= (uint32_t)(4 * q) << (8 * jj);
        }
        o.w[m] = word;
    }
    return o;
}

// Column offsets of a narrow panel (Bp < 32) whose table repeats its byte
// groups (column_source<true>): lane l reads copy (l / Bp) mod floor(32/Bp),
// so byte j of word m = 4 * ((l mod Bp + u) mod Bp + Bp * copy) for position
// u = 4m + j < Bp; positions past Bp are not looked up.
__device__ __noinline__ Offsets narrow_offsets_dup(int lane, int Bp) {
    Offsets o;
    const int copies = 32 / Bp, r = lane % Bp, base = Bp * ((lane / Bp) % copies);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        uint32_t word = 0;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int u = 4 * m + jj;
            int q = r + u;
            q = q >= Bp ? q - Bp : q;
            q = u < Bp ? base + q : 0;
            word |= (uint32_t)(4 * q) << (8 * jj);
        }
        o.w[m] = word;
    }
    return o;
}

// lookup_row over the first nwords stored words only (a narrow panel: its Bp
// = 4 * nwords positions), in lookup_row's order.
__device__ __forceinline__ float lookup_row_narrow(const uint32_t (&w)[8], const uint32_t (&offp)[8],
                                                   const float *tbl, int nwords) {
    unsigned long long acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        if (m < nwords) {
            const float v0 = lds(tbl, prmt(w[m], offp[m], addr_sel(0)));
            const float v1 = lds(tbl, prmt(w[m], offp[m], addr_sel(1)));
            const float v2 = lds(tbl, prmt(w[m], offp[m], addr_sel(2)));
            const float v3 = lds(tbl, prmt(w[m], offp[m], addr_sel(3)));
            acc[(2 * m) & 3] = fadd2(acc[(2 * m) & 3], f2pack(v0, v1));
            acc[(2 * m + 1) & 3] = fadd2(acc[(2 * m + 1) & 3], f2pack(v2, v3));
        }
    }
    return __fadd_rn(__fadd_rn(f2sum(acc[0]), f2sum(acc[1])), __fadd_rn(f2sum(acc[2]), f2sum(acc[3])));
}

// Sum of the byte-table entries selected by one row's 32 stored bytes.  w
// holds position u in byte u%4 of w[u/4]; offp holds, in the same places,
// the byte offset 4*q of the column group each position maps to.
__device__ __forceinline__ float lookup_row(const uint32_t (&w)[8], const uint32_t (&offp)[8], const float *tbl) {
    unsigned long long acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float v0 = lds(tbl, prmt(w[m], offp[m], addr_sel(0)));
        const float v1 = lds(tbl, prmt(w[m], offp[m], addr_sel(1)));
        const float v2 = lds(tbl, prmt(w[m], offp[m], addr_sel(2)));
        const float v3 = lds(tbl, prmt(w[m], offp[m], addr_sel(3)));
        acc[(2 * m) & 3] = fadd2(acc[(2 * m) & 3], f2pack(v0, v1));
        acc[(2 * m + 1) & 3] = fadd2(acc[(2 * m + 1) & 3], f2pack(v2, v3));
    }
    return __fadd_rn(__fadd_rn(f2sum(acc[0]), f2sum(acc[1])), __fadd_rn(f2sum(acc[2]), f2sum(acc[3])));
}

// Two rows' lookups interleaved (twice the independent shared loads in
// flight); each sum is accumulated in the same order as lookup_row's.
__device__ __forceinline__ void lookup_rows2(const uint32_t (&wa)[8], const uint32_t (&wb)[8],
                                             const uint32_t (&offp)[8], const float *tbl, float &sa, float &sb) {
    unsigned long long acc_a[4] = {0, 0, 0, 0}, acc_b[4] = {0, 0, 0, 0};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float a0 = lds(tbl, prmt(wa[m], offp[m], addr_sel(0)));
        const float b0 = lds(tbl, prmt(wb[m], offp[m], addr_sel(0)));
        const float a1 = lds(tbl, prmt(wa[m], offp[m], addr_sel(1)));
        const float b1 = lds(tbl, prmt(wb[m], offp[m], addr_sel(1)));
        const float a2 = lds(tbl, prmt(wa[m], offp[m], addr_sel(2)));
        const float b2 = lds(tbl, prmt(wb[m], offp[m], addr_sel(2)));
        const float a3 = lds(tbl, prmt(wa[m], offp[m], addr_sel(3)));
        const float b3 = lds(tbl, prmt(wb[m], offp[m], addr_sel(3)));
        acc_a[(2 * m) & 3] = fadd2(acc_a[(2 * m) & 3], f2pack(a0, a1));
        acc_b[(2 * m) & 3] = fadd2(acc_b[(2 * m) & 3], f2pack(b0, b1));
        acc_a[(2 * m + 1) & 3] = fadd2(acc_a[(2 * m + 1) & 3], f2pack(a2, a3));
        acc_b[(2 * m + 1) & 3] = fadd2(acc_b[(2 * m + 1) & 3], f2pack(b2, b3));
    }
    sa = __fadd_rn(__fadd_rn(f2sum(acc_a[0]), f2sum(acc_a[1])), __fadd_rn(f2sum(acc_a[2]), f2sum(acc_a[3])));
    sb = __fadd_rn(__fadd_rn(f2sum(acc_b[0]), f2sum(acc_b[1])), __fadd_rn(f2sum(acc_b[2]), f2sum(acc_b[3])));
}

// LUT-BSF for one virtual panel, built by the whole CTA: lane q builds byte
// group q (columns 8q .. 8q+7, z in zp), warp w its entries b = 32w .. 32w+31:
// entry b = T_lo[b & 15] + T_hi[b >> 4], where T_lo and T_hi are the 16-entry
// tables of the group's low and high 4 columns, each (+-z0 +- z1) + (+-z2 +-
// z3).  Columns past a narrow panel's width have z = 0, so their entries are
// 0.  T points at the buffer (entry b of group q at T[b*64 + q]).  Each of
// the NW warps writes 256 / NW consecutive entries b of every group.
template <int NW>
__device__ __forceinline__ void build_byte_table(const float *zp, float *T, int warp, int lane) {
    constexpr int kHi = 16 / NW;   // high-nibble values per warp: entries b = 16*kHi*warp ...
    const float4 za = *reinterpret_cast<const float4 *>(zp + 8 * lane);
    const float4 zb = *reinterpret_cast<const float4 *>(zp + 8 * lane + 4);
    float lo[16];
    sums16(za.x, za.y, za.z, za.w, lo);
    float hi[kHi];
#pragma unroll
    for (int s2 = 0; s2 < kHi; ++s2) {
        const int h = kHi * warp + s2;
        const float s01 = __fadd_rn((h & 1) ? zb.x : -zb.x, (h & 2) ? zb.y : -zb.y);
        const float s23 = __fadd_rn((h & 4) ? zb.z : -zb.z, (h & 8) ? zb.w : -zb.w);
        hi[s2] = __fadd_rn(s01, s23);
    }
    float *col = T + (16 * kHi * warp) * 64 + lane;
#pragma unroll
    for (int s2 = 0; s2 < kHi; ++s2)
#pragma unroll
        for (int v = 0; v < 16; ++v) col[(16 * s2 + v) * 64] = __fadd_rn(lo[v], hi[s2]);
}

// Set (bit 0) when a kernel gave up waiting for a weight copy; the rows of
// that CTA are then written as NaN.  Read and cleared by fb_device_errors.
__device__ unsigned int g_error_flags;

// The row's words of one item of a narrow panel (Bp < 32) from its slot
// (the block's bytes in the packed layout); positions past Bp are zero.
struct Words {
    uint32_t w[8];
};
__device__ __noinline__ Words read_item_narrow(const uint8_t *slot, int Bp, int lane) {
    Words r;
#pragma unroll
    for (int m = 0; m < 8; ++m) r.w[m] = 0;
    if (Bp == 16) {
        const uint4 x0 = *reinterpret_cast<const uint4 *>(slot + 16 * lane);
        r.w[0] = x0.x; r.w[1] = x0.y; r.w[2] = x0.z; r.w[3] = x0.w;
    } else {
#pragma unroll
        for (int m = 0; m < 7; ++m)
            if (m < Bp / 4) r.w[m] = *reinterpret_cast<const uint32_t *>(slot + 128 * m + 4 * lane);
    }
    return r;
}

// The row's words of one item of a full panel from its slot.
__device__ __forceinline__ void read_item_full(const uint8_t *slot, int lane, uint32_t (&w)[8]) {
    const uint4 x0 = *reinterpret_cast<const uint4 *>(slot + 16 * lane);
    const uint4 x1 = *reinterpret_cast<const uint4 *>(slot + 512 + 16 * lane);
    w[0] = x0.x; w[1] = x0.y; w[2] = x0.z; w[3] = x0.w;
    w[4] = x1.x; w[5] = x1.y; w[6] = x1.z; w[7] = x1.w;
}

// Shared-memory layout of one CTA (bytes): two interleaved byte tables |
// z of two panels | kSlots weight slots of cpb KiB | row scales [KB][R] |
// row partials [R] | cluster inbox [R + C].
constexpr int kTableBytes = 65536;
constexpr int kZBytes = 2 * kPanelCols * 4;
constexpr int kItemsPerWarp = 2;

template <int XT, int NW>
__global__ void __launch_bounds__(NW * 32, Shape<NW>::kMinBlocks) gemv_kernel(const __grid_constant__ GemvArgs args) {
    constexpr int kNW = NW, kSlots = Shape<NW>::kSlots;
    extern __shared__ __align__(128) float smem_f[];
    __shared__ __align__(8) unsigned long long s_bar[kSlots];
    // The launch's parameter block is new to every SM's constant cache, and the
    // kernel would touch its fields one after another, each a miss; one
    // parallel copy into shared memory pays that latency once.
    __shared__ __align__(16) GemvArgs s_args;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // (the per-matrix table of grouped calls stays in the parameter block)
    static_assert(offsetof(GemvArgs, mats) % 4 == 0, "parameter block copied as words");
    for (int i = tid; i < (int)(offsetof(GemvArgs, mats) / 4); i += blockDim.x)
        reinterpret_cast<int *>(&s_args)[i] = reinterpret_cast<const int *>(&args)[i];
    if (tid == 0) {
#pragma unroll
        for (int s2 = 0; s2 < kSlots; ++s2) mbar_init(smem_addr(&s_bar[s2]));
        mbar_init_fence();
    }
    if (args.group > 1) {   // a grouped call: this CTA's matrix
        __syncthreads();
        if (tid == 0) {
            int m = 0;
            while (m + 1 < s_args.group && (int)blockIdx.y >= s_args.rb_start[m + 1]) ++m;
            const GemvArgs::Mat &mt = args.mats[m];
            s_args.planes = mt.planes;
            s_args.alpha_r = mt.alpha_r;
            s_args.alpha_c = mt.alpha_c;
            s_args.s_planes = mt.s_planes;
            s_args.s_alpha_r = mt.s_alpha_r;
            s_args.s_alpha_c = mt.s_alpha_c;
            s_args.s_idx = mt.s_idx;
            s_args.y = mt.y;
            s_args.M = mt.M;
            s_args.M_pad = mt.M_pad;
            s_args.nchunks = mt.nchunks;
            s_args.rb_base = s_args.rb_start[m];
        }
    }
    __syncthreads();
    const GemvArgs &a = s_args;
    cg::cluster_group cluster = cg::this_cluster();
    const int j = (int)cluster.block_rank();
    const int rb = (int)blockIdx.y - a.rb_base, b = blockIdx.z;
    const int vb = a.vsplit[j], n_v = a.vsplit[j + 1] - a.vsplit[j];
    const int cpb = a.cpb, R = cpb * kChunkRows;
    const int c_first = rb * cpb;
    const int nvalid = min(cpb, a.nchunks - c_first);   // chunks of this row block inside the matrix
    const int KB = a.K + a.Ks;                          // bases with row scales: global, then salient
    const bool independent = (a.flags & FB_GEMV_INDEPENDENT) != 0;
    const size_t xoff = (size_t)b * a.ldx;
    const int slot_bytes = cpb * 1024;

    float *tables = smem_f;
    float *zbuf = smem_f + kTableBytes / 4;
    uint8_t *slots = reinterpret_cast<uint8_t *>(smem_f) + kTableBytes + kZBytes;
    float *s_ar = reinterpret_cast<float *>(slots + kSlots * slot_bytes);
    float *pw = s_ar + KB * R;
    float *part = pw + R;
    PanelDesc *s_desc = reinterpret_cast<PanelDesc *>(part + ((R + kMaxCluster + 1) & ~1));
    const uint32_t slots_s = smem_addr(slots), bar_s = smem_addr(&s_bar[0]);

    // ---- 1. weight copies and row scales, before the wait -------------------
    // Panel vi's blocks of this row block are contiguous: one bulk copy into
    // slot vi % kSlots, issued by thread 0 kSlots - 1 panels ahead of use.
    uint32_t pending = 0, pend_par = 0;   // thread 0: slots with a copy in flight, its phase parity
    auto issue = [&](int vi, const PanelDesc &d) {
        if (a.flags & FB_GEMV_TEST_WAIT_TIMEOUT) return;   // tests: no copy, so every wait for one runs out
        const int s2 = vi % kSlots;
        const uint32_t blk = 32u * (uint32_t)desc_bp(d);
        bulk_load(slots_s + s2 * slot_bytes, d.pl + (size_t)blk * c_first, blk * (uint32_t)nvalid, bar_s + 8 * s2);
        pending |= 1u << s2;
        pend_par = (pend_par & ~(1u << s2)) | ((uint32_t)(vi / kSlots) & 1u) << s2;
    };
    if (tid == 0)
        for (int v = 0; v < kSlots - 1 && v < n_v; ++v) issue(v, panel_desc(a, vb + v));
    for (int t = tid; t < n_v; t += blockDim.x) s_desc[t] = panel_desc(a, vb + t);

    // column data of one panel: thread t stages column t
    // Two register sets, for panels of even and odd index: panel p is staged
    // two panels before its z is written (the loop below is unrolled by two,
    // so the set is chosen at compile time).
    struct Staged {
        float ac;
        uint32_t x;
        int xi;
    };
    Staged st[2] = {{0.0f, 0u, -1}, {0.0f, 0u, -1}};
    auto stage = [&](Staged &t, const PanelDesc &d, bool read_x) {
        t.x = 0;
        if (tid >= kPanelCols) return;
        column_source(a, d, tid, t.ac, t.xi);
        if (read_x && t.xi >= 0) t.x = load_x_bits<XT>(a.x, xoff + t.xi);
    };
    auto z_of = [&](const Staged &t) { return t.xi >= 0 ? __fmul_rn(t.ac, x_value<XT>(t.x)) : 0.0f; };
    if (n_v > 0) stage(st[0], panel_desc(a, vb), independent);
    griddep_launch_dependents();
    // the row block's row scales, every base (rows past M: 0); a thread's
    // loads are issued in batches of kArBatch before any is stored, so they
    // cost one memory latency per batch rather than one each
    constexpr int kArBatch = 8;
    for (int t0 = 0; t0 < KB * R; t0 += kArBatch * (int)blockDim.x) {
        float v[kArBatch];
#pragma unroll
        for (int u = 0; u < kArBatch; ++u) {
            const int t = t0 + u * (int)blockDim.x + tid;
            const int kb = t / R, r = t - kb * R, row = c_first * kChunkRows + r;
            const float *src = row_scales(a, kb);
            v[u] = t < KB * R && row < a.M ? __ldg(src + row) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kArBatch; ++u) {
            const int t = t0 + u * (int)blockDim.x + tid;
            if (t < KB * R) s_ar[t] = v[u];
        }
    }

    // ---- 2. activations (may be the previous kernel's output) --------------
    if (!independent) {
        griddep_wait();
        if (st[0].xi >= 0) st[0].x = load_x_bits<XT>(a.x, xoff + st[0].xi);
    }
    if (tid < kPanelCols) zbuf[tid] = z_of(st[0]);
    __syncthreads();   // z of panel 0, panel descriptors and row scales written
    if (n_v > 1) stage(st[1], s_desc[1], true);
    if (n_v > 2) stage(st[0], s_desc[2], true);

    // column offsets of a full panel (narrow panels compute theirs)
    uint32_t off_full[8];
    full_offsets(lane, off_full);

    // ---- 3. per panel: its byte tables, then this warp's chunks -------------
    // Warp w owns chunks w + kNW * i of the row block; each lane keeps its
    // rows' partial sums and current row scales in registers.  The barrier of
    // panel vi also ends every warp's reads of panel vi - 1, whose slot then
    // takes panel vi + kSlots - 1.
    bool failed = false;
    float racc[kItemsPerWarp], rar[kItemsPerWarp];
#pragma unroll
    for (int it = 0; it < kItemsPerWarp; ++it) racc[it] = rar[it] = 0.0f;
    int kb_cur = -1, sl = 0;   // sl = vi % kSlots
    // One panel; the table buffer is a compile-time constant in each of the
    // two copies, so table addresses fold into the shared loads.
    auto panel = [&](auto bufc, int vi) {
        constexpr int buf = decltype(bufc)::value;
        const int Bp = desc_bp(s_desc[vi]), kb = s_desc[vi].kb;
        bool ok = !failed;
        if (ok) {
            const uint32_t par = (uint32_t)(vi / kSlots) & 1u;
            ok = mbar_try_wait(bar_s + 8 * sl, par) || mbar_wait_bounded(bar_s + 8 * sl, par);
        }
        if (tid == 0 && ok) pending &= ~(1u << sl);
        float *tb = tables + 32 * buf;
        build_byte_table<NW>(zbuf + buf * kPanelCols, tb, warp, lane);
        if (vi + 1 < n_v && tid < kPanelCols)   // z of the next panel into the other buffer
            zbuf[(buf ^ 1) * kPanelCols + tid] = z_of(st[buf ^ 1]);
        if (vi + 3 < n_v) stage(st[buf ^ 1], s_desc[vi + 3], true);
        // tables of panel vi complete; every warp done with panel vi - 1
        failed = __syncthreads_or(!ok) != 0;
        if (failed) return;
        if (tid == 0 && vi + kSlots - 1 < n_v) issue(vi + kSlots - 1, s_desc[vi + kSlots - 1]);
        if (kb != kb_cur) {   // a new base: its row scales
            kb_cur = kb;
#pragma unroll
            for (int it = 0; it < kItemsPerWarp; ++it) {
                const int cl = warp + kNW * it;
                if (cl < cpb) rar[it] = s_ar[kb_cur * R + cl * kChunkRows + lane];
            }
        }
        const uint8_t *slot = slots + sl * slot_bytes;
        sl = sl + 1 == kSlots ? 0 : sl + 1;
        static_assert(kItemsPerWarp == 2, "the full-panel path looks up a warp's two items together");
        if (Bp == 32 && warp + kNW < nvalid) {   // both items: interleaved
            uint32_t w0[8], w1[8];
            read_item_full(slot + warp * 1024, lane, w0);
            read_item_full(slot + (warp + kNW) * 1024, lane, w1);
            float s0, s1;
            lookup_rows2(w0, w1, off_full, tb, s0, s1);
            racc[0] = __fadd_rn(racc[0], __fmul_rn(rar[0], s0));
            racc[1] = __fadd_rn(racc[1], __fmul_rn(rar[1], s1));
        } else if (Bp == 32) {
            if (warp < nvalid) {
                uint32_t w[8];
                read_item_full(slot + warp * 1024, lane, w);
                racc[0] = __fadd_rn(racc[0], __fmul_rn(rar[0], lookup_row(w, off_full, tb)));
            }
        } else {
            const Offsets o = narrow_offsets(lane, Bp);
#pragma unroll 1
            for (int it = 0; it < kItemsPerWarp; ++it) {
                const int cl = warp + kNW * it;
                if (cl < nvalid) {
                    const Words r = read_item_narrow(slot + cl * 32 * Bp, Bp, lane);
                    const float sum = lookup_row(r.w, o.w, tb);
#pragma unroll
                    for (int i2 = 0; i2 < kItemsPerWarp; ++i2)
                        if (i2 == it) racc[i2] = __fadd_rn(racc[i2], __fmul_rn(rar[i2], sum));
                }
            }
        }
    };
#pragma unroll 1
    for (int vi = 0; vi < n_v; vi += 2) {
        panel(std::integral_constant<int, 0>{}, vi);
        if (vi + 1 < n_v) panel(std::integral_constant<int, 1>{}, vi + 1);
    }
#pragma unroll
    for (int it = 0; it < kItemsPerWarp; ++it) {
        const int cl = warp + kNW * it;
        if (cl < cpb) pw[cl * kChunkRows + lane] = racc[it];
    }
    if (failed && tid == 0) {
        // Wait (bounded) for the copies still in flight, so none lands after
        // the CTA has gone, then flag the failure.
        for (int s2 = 0; s2 < kSlots; ++s2)
            if (pending & (1u << s2)) mbar_wait_bounded(bar_s + 8 * s2, (pend_par >> s2) & 1u);
        atomicOr(&g_error_flags, 1u);
    }

    // ---- 4. the cluster's row partials, in a fixed order --------------------
    // Rows are owned in runs of Rq: rank o sums rows [o*Rq, min((o+1)*Rq, R)).
    // Every CTA pushes its row partials into the owner's inbox (slot = its
    // own rank), one cluster barrier makes them visible, and each owner adds
    // its inbox in rank order.  After the barrier no CTA touches another's
    // shared memory, so none has to wait for the others before exiting.
    const int Rq = (R + a.C - 1) / a.C;
    __syncthreads();
    for (int r = tid; r < R; r += blockDim.x) {
        const float sum = failed ? __int_as_float(0x7fc00000) : pw[r];
        const int owner = r / Rq;
        float *inbox = cluster.map_shared_rank(part, owner);
        inbox[j * Rq + (r - owner * Rq)] = sum;
    }
    cluster.sync();
    for (int i = tid; i < Rq; i += blockDim.x) {
        const int r = j * Rq + i;
        if (r >= R) break;
        float sum = part[i];
        for (int jj = 1; jj < a.C; ++jj) sum = __fadd_rn(sum, part[jj * Rq + i]);
        const int row = c_first * kChunkRows + r;
        if (row < a.M) a.y[(size_t)b * a.ldy + row] = sum;
    }
    if (independent) griddep_wait();   // complete only after the previous kernel
}

// ---- The streaming kernel: weights straight into registers --------------
//
// Same work units, tables, lookups and cluster reduction as gemv_kernel, but
// the packed weights are not staged in shared memory: each lane loads its
// rows' words of the panel after next with 128-bit loads into one of two
// register sets while it looks up the current panel from the other, so a
// weight byte costs shared-memory bandwidth only for its table lookup.  8
// warps per CTA and about 70 KB of shared memory let two CTAs share an SM,
// so one CTA's prologue, barriers and reduction overlap the other's
// lookups.  For calls that depend on the previous kernel the first two
// panels' words (and an L2 prefetch of the rest of the slice) are requested
// before the programmatic-launch wait.

// 16 bytes of packed weights, read once: not kept in L1.
__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ldg_stream32(const void *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// This lane's words of one item of a narrow panel (Bp < 32) in global
// memory; positions past Bp are zero.
__device__ __noinline__ Words load_item_narrow(const uint8_t *blk, int Bp, int lane) {
    Words r;
#pragma unroll
    for (int m = 0; m < 8; ++m) r.w[m] = 0;
    if (Bp == 16) {
        const uint4 x0 = ldg_stream(blk + 16 * lane);
        r.w[0] = x0.x; r.w[1] = x0.y; r.w[2] = x0.z; r.w[3] = x0.w;
    } else {
#pragma unroll
        for (int m = 0; m < 7; ++m)
            if (m < Bp / 4) r.w[m] = ldg_stream32(blk + 128 * m + 4 * lane);
    }
    return r;
}

constexpr int kStreamWarps = 8;
constexpr int kDescRing = 8;   // panel descriptors kept in shared memory (a ring)

template <int XT, int I>
__global__ void __launch_bounds__(kStreamWarps * 32, 2) stream_kernel(const __grid_constant__ GemvArgs args) {
    constexpr int NW = kStreamWarps;
    extern __shared__ __align__(128) float smem_f[];
    __shared__ __align__(16) GemvArgs s_args;
    __shared__ __align__(16) PanelDesc s_ring[kDescRing];
    __shared__ __align__(8) unsigned long long s_inbox_bar;   // the cluster's row partials have landed
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    static_assert(offsetof(GemvArgs, mats) % 4 == 0, "parameter block copied as words");
    for (int i = tid; i < (int)(offsetof(GemvArgs, mats) / 4); i += blockDim.x)
        reinterpret_cast<int *>(&s_args)[i] = reinterpret_cast<const int *>(&args)[i];
    if (args.group > 1) {   // a grouped call: this CTA's matrix
        __syncthreads();
        if (tid == 0) {
            int m = 0;
            while (m + 1 < s_args.group && (int)blockIdx.y >= s_args.rb_start[m + 1]) ++m;
            const GemvArgs::Mat &mt = args.mats[m];
            s_args.planes = mt.planes;
            s_args.alpha_r = mt.alpha_r;
            s_args.alpha_c = mt.alpha_c;
            s_args.s_planes = mt.s_planes;
            s_args.s_alpha_r = mt.s_alpha_r;
            s_args.s_alpha_c = mt.s_alpha_c;
            s_args.s_idx = mt.s_idx;
            s_args.y = mt.y;
            s_args.M = mt.M;
            s_args.M_pad = mt.M_pad;
            s_args.nchunks = mt.nchunks;
            s_args.rb_base = s_args.rb_start[m];
        }
    }
    __syncthreads();
    const GemvArgs &a = s_args;
    cg::cluster_group cluster = cg::this_cluster();
    const int j = (int)cluster.block_rank();
    const int rb = (int)blockIdx.y - a.rb_base, b = blockIdx.z;
    const int vb = a.vsplit[j], n_v = a.vsplit[j + 1] - a.vsplit[j];
    const int cpb = a.cpb, R = cpb * kChunkRows;
    const int c_first = rb * cpb;
    const int nvalid = min(cpb, a.nchunks - c_first);
    const bool independent = (a.flags & FB_GEMV_INDEPENDENT) != 0;
    const size_t xoff = (size_t)b * a.ldx;

    float *tables = smem_f;
    float *zbuf = smem_f + kTableBytes / 4;
    float *part = zbuf + 2 * kPanelCols;   // cluster inbox: R + C floats

    griddep_launch_dependents();
    // The row partials reach their owner CTA as asynchronous remote stores
    // that complete on the owner's inbox barrier: it expects C * (its rows)
    // * 4 bytes (its own slot included).  The barrier is initialised and its
    // bytes announced before the cluster arrive; every CTA waits for that
    // arrive just before its first remote store.
    const int Rq = (R + a.C - 1) / a.C;
    const uint32_t inbox_bar = smem_addr(&s_inbox_bar);
    if (tid == 0) {
        mbar_init(inbox_bar);
        mbar_init_fence();
        const int owned = max(0, min(Rq, R - j * Rq));
        mbar_arrive_expect(inbox_bar, (uint32_t)(a.C * owned * 4));
    }
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

    // ---- 1. before the wait: the first two panels' words, their row
    // scales, the column sources of panel 0 (and its x when independent) --
    uint32_t wA[I][8], wB[I][8];
    float rarA[I], rarB[I];
    auto load_panel = [&](uint32_t (&w)[I][8], float (&rar)[I], const PanelDesc &d) {
        const int Bp = desc_bp(d);
        const size_t blk = 32u * (unsigned)Bp;
        const float *src = row_scales(a, d.kb);
#pragma unroll
        for (int i = 0; i < I; ++i) {
            const int cl = warp + NW * i;
            const int row = (c_first + cl) * kChunkRows + lane;
            rar[i] = cl < nvalid && row < a.M ? __ldg(src + row) : 0.0f;
            if (cl < nvalid) {
                const uint8_t *p = d.pl + blk * (size_t)(c_first + cl);
                if (Bp == 32) {
                    const uint4 x0 = ldg_stream(p + 16 * lane), x1 = ldg_stream(p + 512 + 16 * lane);
                    w[i][0] = x0.x; w[i][1] = x0.y; w[i][2] = x0.z; w[i][3] = x0.w;
                    w[i][4] = x1.x; w[i][5] = x1.y; w[i][6] = x1.z; w[i][7] = x1.w;
                } else {
                    const Words r = load_item_narrow(p, Bp, lane);
#pragma unroll
                    for (int m = 0; m < 8; ++m) w[i][m] = r.w[m];
                }
            }
        }
    };
    if (tid < kDescRing - 4 && tid < n_v) s_ring[tid] = panel_desc(a, vb + tid);
    struct Staged {
        float ac;
        uint32_t x;
        int xi;
    };
    Staged st[2] = {{0.0f, 0u, -1}, {0.0f, 0u, -1}};
    auto stage = [&](Staged &t, const PanelDesc &d, bool read_x) {
        t.x = 0;
        column_source<true>(a, d, tid, t.ac, t.xi);
        if (read_x && t.xi >= 0) t.x = load_x_bits<XT>(a.x, xoff + t.xi);
    };
    auto z_of = [&](const Staged &t) { return t.xi >= 0 ? __fmul_rn(t.ac, x_value<XT>(t.x)) : 0.0f; };
    PanelDesc d1;
    if (n_v > 0) {
        const PanelDesc d0 = panel_desc(a, vb);
        load_panel(wA, rarA, d0);
        stage(st[0], d0, independent);
    }
    if (n_v > 1) {
        d1 = panel_desc(a, vb + 1);
        load_panel(wB, rarB, d1);
    }
    if (!independent) {
        // the rest of the slice into L2 while the previous kernel finishes
        if (tid == 0) {
            for (int v = 2; v < min(n_v, 8); ++v) {
                const PanelDesc d = panel_desc(a, vb + v);
                const uint32_t blk = 32u * (uint32_t)desc_bp(d);
                prefetch_l2(d.pl + (size_t)blk * c_first, blk * (uint32_t)nvalid);
            }
        }
        griddep_wait();
        if (st[0].xi >= 0) st[0].x = load_x_bits<XT>(a.x, xoff + st[0].xi);
    }
    if (n_v > 1) stage(st[1], d1, true);   // x of panel 1 in flight with panel 0's
    zbuf[tid] = z_of(st[0]);
    __syncthreads();   // z of panel 0 and the first descriptors written
    if (n_v > 2) stage(st[0], s_ring[2], true);

    uint32_t off_full[8];
    full_offsets(lane, off_full);

    float racc[I];
#pragma unroll
    for (int i = 0; i < I; ++i) racc[i] = 0.0f;

    // ---- 2. per panel: tables, then this warp's items ----------------------
    auto panel = [&](auto bufc, int vi, uint32_t (&w)[I][8], float (&rar)[I]) {
        constexpr int buf = decltype(bufc)::value;
        const int Bp = desc_bp(s_ring[vi % kDescRing]);
        float *tb = tables + 32 * buf;
        build_byte_table<NW>(zbuf + buf * kPanelCols, tb, warp, lane);
        if (vi + 1 < n_v) zbuf[(buf ^ 1) * kPanelCols + tid] = z_of(st[buf ^ 1]);
        if (vi + 3 < n_v) stage(st[buf ^ 1], s_ring[(vi + 3) % kDescRing], true);
        if (tid == 0 && vi + 4 < n_v) s_ring[(vi + 4) % kDescRing] = panel_desc(a, vb + vi + 4);
        __syncthreads();   // tables of panel vi complete; every warp done with panel vi - 1
        if (Bp == 32) {
#pragma unroll
            for (int i = 0; i < I; i += 2) {
                const int c0 = warp + NW * i;
                if (i + 1 < I && c0 + NW < nvalid) {
                    float s0, s1;
                    lookup_rows2(w[i], w[i + 1], off_full, tb, s0, s1);
                    racc[i] = __fadd_rn(racc[i], __fmul_rn(rar[i], s0));
                    racc[i + 1] = __fadd_rn(racc[i + 1], __fmul_rn(rar[i + 1], s1));
                } else if (c0 < nvalid) {
                    racc[i] = __fadd_rn(racc[i], __fmul_rn(rar[i], lookup_row(w[i], off_full, tb)));
                }
            }
        } else {
            const Offsets o = narrow_offsets_dup(lane, Bp);
#pragma unroll
            for (int i = 0; i < I; ++i)
                if (warp + NW * i < nvalid)
                    racc[i] = __fadd_rn(racc[i], __fmul_rn(rar[i], lookup_row_narrow(w[i], o.w, tb, Bp >> 2)));
        }
        if (vi + 2 < n_v) load_panel(w, rar, s_ring[(vi + 2) % kDescRing]);
    };
#pragma unroll 1
    for (int vi = 0; vi < n_v; vi += 2) {
        panel(std::integral_constant<int, 0>{}, vi, wA, rarA);
        if (vi + 1 < n_v) panel(std::integral_constant<int, 1>{}, vi + 1, wB, rarB);
    }

    // ---- 3. the cluster's row partials, summed by their owner in rank order
    // Rows are owned in runs of Rq: rank o sums rows [o*Rq, min((o+1)*Rq, R)).
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (!(a.flags & FB_GEMV_TEST_WAIT_TIMEOUT)) {   // (tests: nothing is pushed, so the wait runs out)
#pragma unroll
        for (int i = 0; i < I; ++i) {
            const int r = (warp + NW * i) * kChunkRows + lane;
            if (warp + NW * i < cpb) {
                const int owner = r / Rq;
                push_remote(smem_addr(part + j * Rq + (r - owner * Rq)), inbox_bar, owner, racc[i]);
            }
        }
    }
    const bool ok = mbar_try_wait_cluster(inbox_bar, 0) || mbar_wait_bounded<true>(inbox_bar, 0);
    if (!ok && tid == 0) atomicOr(&g_error_flags, 1u);
    for (int i = tid; i < Rq; i += blockDim.x) {
        const int r = j * Rq + i;
        if (r >= R) break;
        float sum = part[i];
        for (int jj = 1; jj < a.C; ++jj) sum = __fadd_rn(sum, part[jj * Rq + i]);
        const int row = c_first * kChunkRows + r;
        if (row < a.M) a.y[(size_t)b * a.ldy + row] = ok ? sum : __int_as_float(0x7fc00000);
    }
    if (independent) griddep_wait();   // complete only after the previous kernel
}

// ---- The batched kernel: one weight pass for up to 16 tokens -------------
//
// Several activation vectors share each weight word: a CTA loads a panel's
// words for its rows into registers once (two register sets, the panel after
// next loading while the current one is used) and applies them to the
// tables of every token of its pass, two tokens at a time.  The two tokens'
// tables share each 256-byte row: entry b of byte group q is at b*256 + 4q
// for the first token and at b*256 + 128 + 4q for the second, so both
// lookups of a weight byte use one address (the second at a constant +128),
// and the column offset stays below 128 (the sign-replicating byte select of
// the address needs that).  Per token, every sum is formed in exactly the
// order the batch-1 kernels use, and the per-token row partials are kept in
// shared memory (any number of tokens per pass).
//
// Shared memory: two table buffers of 64 KB (after the last lookups, the
// same bytes receive the cluster's row partials) | z of two steps (2
// tokens x 256 columns each) | row partials [tp][R].
constexpr int kBatchWarps = 16;
constexpr int kMaxTokensPerPass = 16;
constexpr int kPairTableBytes = 65536;

// The two tokens' sums of the entries selected by one row's stored bytes,
// each in lookup_row's order: eight chains (accumulator k = (2m + j/2) & 3,
// half j & 1), then per token (lo + hi) of each k, then (k0 + k1) + (k2 + k3).
// (nwords < 8: a narrow panel, only its first nwords stored words.)
__device__ __forceinline__ void lookup_row_t2(const uint32_t (&w)[8], const uint32_t (&offp)[8], const float *tbl,
                                              float &s0, float &s1, int nwords = 8) {
    unsigned long long acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        if (m >= nwords) break;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const uint32_t off = prmt(w[m], offp[m], addr_sel(jj));
            const unsigned long long v = f2pack(lds(tbl, off), lds(tbl + 32, off));
            const int slot = 2 * ((2 * m + (jj >> 1)) & 3) + (jj & 1);
            acc[slot] = fadd2(acc[slot], v);
        }
    }
    const unsigned long long p0 = fadd2(acc[0], acc[1]), p1 = fadd2(acc[2], acc[3]);
    const unsigned long long p2 = fadd2(acc[4], acc[5]), p3 = fadd2(acc[6], acc[7]);
    const unsigned long long r = fadd2(fadd2(p0, p1), fadd2(p2, p3));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(s0), "=f"(s1) : "l"(r));
}

// LUT-BSF for one panel and two tokens, built by the whole CTA (16 warps):
// lane q builds byte group q, warp w the entries b = 16w .. 16w + 15 of both
// tokens (z of token t at zp + 256t); entry b = T_lo[b & 15] + T_hi[b >> 4]
// per token, as build_byte_table; token t's entries at +128t in each row.
__device__ __forceinline__ void build_pair_table(const float *zp, float *T, int warp, int lane) {
    float lo0[16], lo1[16];
    {
        const float4 za = *reinterpret_cast<const float4 *>(zp + 8 * lane);
        sums16(za.x, za.y, za.z, za.w, lo0);
        const float4 zc = *reinterpret_cast<const float4 *>(zp + kPanelCols + 8 * lane);
        sums16(zc.x, zc.y, zc.z, zc.w, lo1);
    }
    const int h = warp;   // the high nibble of this warp's entries
    const float4 zb = *reinterpret_cast<const float4 *>(zp + 8 * lane + 4);
    const float4 zd = *reinterpret_cast<const float4 *>(zp + kPanelCols + 8 * lane + 4);
    const float hi0 = __fadd_rn(__fadd_rn((h & 1) ? zb.x : -zb.x, (h & 2) ? zb.y : -zb.y),
                                __fadd_rn((h & 4) ? zb.z : -zb.z, (h & 8) ? zb.w : -zb.w));
    const float hi1 = __fadd_rn(__fadd_rn((h & 1) ? zd.x : -zd.x, (h & 2) ? zd.y : -zd.y),
                                __fadd_rn((h & 4) ? zd.z : -zd.z, (h & 8) ? zd.w : -zd.w));
    float *col = T + (16 * h) * 64 + lane;
#pragma unroll
    for (int v = 0; v < 16; ++v) {
        col[v * 64] = __fadd_rn(lo0[v], hi0);
        col[v * 64 + 32] = __fadd_rn(lo1[v], hi1);
    }
}

template <int XT, int I>
__global__ void __launch_bounds__(kBatchWarps * 32, 1) batched_kernel(const __grid_constant__ GemvArgs args) {
    constexpr int NW = kBatchWarps, NT = NW * 32;
    extern __shared__ __align__(128) float smem_f[];
    __shared__ __align__(16) GemvArgs s_args;
    __shared__ __align__(16) PanelDesc s_ring[kDescRing];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < (int)(offsetof(GemvArgs, mats) / 4); i += blockDim.x)
        reinterpret_cast<int *>(&s_args)[i] = reinterpret_cast<const int *>(&args)[i];
    __syncthreads();
    const GemvArgs &a = s_args;
    cg::cluster_group cluster = cg::this_cluster();
    const int j = (int)cluster.block_rank();
    const int rb = (int)blockIdx.y;
    const int vb = a.vsplit[j], n_v = a.vsplit[j + 1] - a.vsplit[j];
    const int cpb = a.cpb, R = cpb * kChunkRows;
    const int c_first = rb * cpb;
    const int nvalid = min(cpb, a.nchunks - c_first);
    const bool independent = (a.flags & FB_GEMV_INDEPENDENT) != 0;
    const int TP = a.tp, t_base = (int)blockIdx.z * TP, nt = min(TP, a.batch - t_base);
    const int npairs = (nt + 1) >> 1, S = n_v * npairs;

    float *tables = smem_f;                                   // 2 x 64 KB
    float *zbuf = smem_f + 2 * kPairTableBytes / 4;           // [2][2][256]
    float *accs = zbuf + 4 * kPanelCols;                      // [TP][R]
    float *inbox = tables;                                    // after the last lookups

    griddep_launch_dependents();
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

    for (int i = tid; i < TP * R; i += NT) accs[i] = 0.0f;
    if (tid < kDescRing - 4 && tid < n_v) s_ring[tid] = panel_desc(a, vb + tid);

    uint32_t wA[I][8], wB[I][8];
    float rarA[I], rarB[I];
    auto load_panel = [&](uint32_t (&w)[I][8], float (&rar)[I], const PanelDesc &d) {
        const int Bp = desc_bp(d);
        const size_t blk = 32u * (unsigned)Bp;
        const float *src = row_scales(a, d.kb);
#pragma unroll
        for (int i = 0; i < I; ++i) {
            const int cl = warp + NW * i;
            const int row = (c_first + cl) * kChunkRows + lane;
            rar[i] = cl < nvalid && row < a.M ? __ldg(src + row) : 0.0f;
            if (cl < nvalid) {
                const uint8_t *p = d.pl + blk * (size_t)(c_first + cl);
                if (Bp == 32) {
                    const uint4 x0 = ldg_stream(p + 16 * lane), x1 = ldg_stream(p + 512 + 16 * lane);
                    w[i][0] = x0.x; w[i][1] = x0.y; w[i][2] = x0.z; w[i][3] = x0.w;
                    w[i][4] = x1.x; w[i][5] = x1.y; w[i][6] = x1.z; w[i][7] = x1.w;
                } else {
                    const Words r = load_item_narrow(p, Bp, lane);
#pragma unroll
                    for (int m = 0; m < 8; ++m) w[i][m] = r.w[m];
                }
            }
        }
    };
    // z staging: thread t stages column t & 255 of token 2*pair + (t >> 8)
    struct Staged {
        float ac;
        uint32_t x;
        int xi;
    };
    Staged st[2] = {{0.0f, 0u, -1}, {0.0f, 0u, -1}};
    const int col = tid & (kPanelCols - 1), half = tid >> 8;
    auto stage = [&](Staged &t, const PanelDesc &d, int pair, bool read_x) {
        t.x = 0;
        const int tok = 2 * pair + half;
        column_source<true>(a, d, col, t.ac, t.xi);
        if (tok >= nt) t.xi = -1;
        if (read_x && t.xi >= 0) t.x = load_x_bits<XT>(a.x, (size_t)(t_base + tok) * a.ldx + t.xi);
    };
    auto z_of = [&](const Staged &t) { return t.xi >= 0 ? __fmul_rn(t.ac, x_value<XT>(t.x)) : 0.0f; };
    auto desc_of_step = [&](int s2) -> const PanelDesc & { return s_ring[(s2 / npairs) % kDescRing]; };

    if (n_v > 0) {
        const PanelDesc d0 = panel_desc(a, vb);
        load_panel(wA, rarA, d0);
        stage(st[0], d0, 0, independent);
    }
    if (n_v > 1) load_panel(wB, rarB, panel_desc(a, vb + 1));
    if (!independent) {
        griddep_wait();
        if (st[0].xi >= 0) st[0].x = load_x_bits<XT>(a.x, (size_t)(t_base + half) * a.ldx + st[0].xi);
    }
    zbuf[tid] = z_of(st[0]);   // step 0 -> z buffer 0
    __syncthreads();
    if (S > 1) stage(st[1], desc_of_step(1), 1 % npairs, true);
    if (S > 2) stage(st[0], desc_of_step(2), 2 % npairs, true);

    uint32_t off_full[8];
    full_offsets(lane, off_full);

    // One step s (panel vi, token pair tp): tables of both tokens into buffer
    // s & 1, z of step s + 1 into the other z buffer, then lookups.
    auto panel = [&](int vi, uint32_t (&w)[I][8], float (&rar)[I]) {
        const int Bp = desc_bp(s_ring[vi % kDescRing]);
        uint32_t offn[8];
        if (Bp != 32) {
            const Offsets o = narrow_offsets_dup(lane, Bp);
#pragma unroll
            for (int m = 0; m < 8; ++m) offn[m] = o.w[m];
        }
#pragma unroll 1
        for (int tp = 0; tp < npairs; ++tp) {
            const int s2 = vi * npairs + tp, buf = s2 & 1;
            float *tb = tables + buf * (kPairTableBytes / 4);
            build_pair_table(zbuf + buf * 2 * kPanelCols, tb, warp, lane);
            if (s2 + 1 < S) zbuf[(buf ^ 1) * 2 * kPanelCols + tid] = z_of(st[(s2 + 1) & 1]);
            if (s2 + 3 < S) stage(st[(s2 + 3) & 1], desc_of_step(s2 + 3), (s2 + 3) % npairs, true);
            if (tid == 0 && tp == 0 && vi + 4 < n_v) s_ring[(vi + 4) % kDescRing] = panel_desc(a, vb + vi + 4);
            __syncthreads();   // tables of step s2 complete; every warp done with step s2 - 1
#pragma unroll
            for (int i = 0; i < I; ++i) {
                const int cl = warp + NW * i;
                if (cl >= nvalid) continue;
                float s0, s1;
                if (Bp == 32)
                    lookup_row_t2(w[i], off_full, tb, s0, s1);
                else
                    lookup_row_t2(w[i], offn, tb, s0, s1, Bp >> 2);
                const int r = cl * kChunkRows + lane;
                float *p0 = accs + (2 * tp) * R + r;
                *p0 = __fadd_rn(*p0, __fmul_rn(rar[i], s0));
                if (2 * tp + 1 < nt) p0[R] = __fadd_rn(p0[R], __fmul_rn(rar[i], s1));
            }
        }
        if (vi + 2 < n_v) load_panel(w, rar, s_ring[(vi + 2) % kDescRing]);
    };
#pragma unroll 1
    for (int vi = 0; vi < n_v; vi += 2) {
        panel(vi, wA, rarA);
        if (vi + 1 < n_v) panel(vi + 1, wB, rarB);
    }

    // ---- the cluster's row partials, per token, in a fixed order ------------
    const int Rq = (R + a.C - 1) / a.C;
    __syncthreads();   // this CTA's lookups are done (its table bytes may be overwritten)
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    cluster.sync();    // every CTA's lookups are done
    for (int e = tid; e < nt * R; e += NT) {
        const int t = e / R, r = e - t * R;
        const int owner = r / Rq;
        float *ib = cluster.map_shared_rank(inbox, owner);
        ib[(j * TP + t) * Rq + (r - owner * Rq)] = accs[t * R + r];
    }
    cluster.sync();
    for (int e = tid; e < nt * Rq; e += NT) {
        const int t = e / Rq, i = e - t * Rq;
        const int r = j * Rq + i;
        if (r >= R) continue;
        float sum = inbox[t * Rq + i];
        for (int jj = 1; jj < a.C; ++jj) sum = __fadd_rn(sum, inbox[(jj * TP + t) * Rq + i]);
        const int row = c_first * kChunkRows + r;
        if (row < a.M) a.y[(size_t)(t_base + t) * a.ldy + row] = sum;
    }
    if (independent) griddep_wait();
}

using KernelFn = void (*)(GemvArgs);

template <int NW>
KernelFn pick_xt(fb_dtype t) {
    return t == FB_F32 ? gemv_kernel<FB_F32, NW> : t == FB_F16 ? gemv_kernel<FB_F16, NW> : gemv_kernel<FB_BF16, NW>;
}

KernelFn pick_kernel(fb_dtype t, int nw) { return nw == 16 ? pick_xt<16>(t) : pick_xt<8>(t); }

template <int I>
KernelFn pick_batched_xt(fb_dtype t) {
    return t == FB_F32 ? batched_kernel<FB_F32, I> : t == FB_F16 ? batched_kernel<FB_F16, I> : batched_kernel<FB_BF16, I>;
}
KernelFn pick_batched(fb_dtype t, int items) { return items == 1 ? pick_batched_xt<1>(t) : pick_batched_xt<2>(t); }

template <int I>
KernelFn pick_stream_xt(fb_dtype t) {
    return t == FB_F32 ? stream_kernel<FB_F32, I> : t == FB_F16 ? stream_kernel<FB_F16, I> : stream_kernel<FB_BF16, I>;
}
KernelFn pick_stream(fb_dtype t, int items) {
    return items == 1 ? pick_stream_xt<1>(t) : items == 2 ? pick_stream_xt<2>(t) : pick_stream_xt<4>(t);
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

struct Plan {
    int M_pad, Pg, Ps, nS_pad, V, nchunks;
    int C, cpb, RB, nwarps;
    int kind;    // 0: gemv_kernel (weights through shared-memory slots); 1: stream_kernel; 2: batched_kernel
    int items;   // stream / batched kernel: chunks per warp per panel
    int tp, passes;   // batched kernel: tokens per pass, passes (grid.z)
    int vsplit[kMaxCluster + 1];
    size_t smem;
};

struct PlanKey {
    int M, N, K, g, nS, Ks, batch, sms, G;
    bool independent, slots;
    bool operator==(const PlanKey &o) const {
        return M == o.M && N == o.N && K == o.K && g == o.g && nS == o.nS && Ks == o.Ks && batch == o.batch &&
               sms == o.sms && G == o.G && independent == o.independent && slots == o.slots;
    }
};

void split_panels(int V, int C, int *vsplit, int *max_n) {
    *max_n = 0;
    for (int jj = 0; jj <= C; ++jj) vsplit[jj] = (int)((long)V * jj / C);
    for (int jj = 0; jj < C; ++jj) *max_n = std::max(*max_n, vsplit[jj + 1] - vsplit[jj]);
}

// Byte groups a CTA looks up per row in each virtual panel (global panels of
// base 0, 1, ..., then salient ones): 32 for a full panel and for every
// half-panel (its other half reads zero entries), the panel's width / 8 for
// a narrow panel.
std::vector<int> vpanel_groups(int N, int K, int hsplit, int nS_pad, int Ks) {
    std::vector<int> g;
    const int Pv = global_vpanels(N, hsplit);
    for (int k = 0; k < K; ++k)
        for (int pp = 0; pp < Pv; ++pp) g.push_back(panel_width(N, hsplit ? pp >> 1 : pp) >> 3);
    if (nS_pad > 0)
        for (int k = 0; k < Ks; ++k)
            for (int p = 0; p < num_panels(nS_pad); ++p) g.push_back(panel_width(nS_pad, p) >> 3);
    return g;
}

// Contiguous split of the virtual panels over C CTAs balancing each CTA's
// shared-memory work: per panel one table build (256 wavefronts) plus cpb
// chunks x its byte groups of lookups.  CTA j takes [vsplit[j], vsplit[j+1]);
// returns the largest CTA's work.
double split_weighted(const std::vector<int> &groups, int C, int cpb, int *vsplit) {
    const int V = (int)groups.size();
    C = std::max(1, std::min(C, V));
    std::vector<double> cost(V);
    double lo = 0.0, hi = 0.0;
    for (int v = 0; v < V; ++v) {
        cost[v] = 256.0 + (double)cpb * groups[v];
        lo = std::max(lo, cost[v]);
        hi += cost[v];
    }
    // the smallest cap under which a greedy fill needs at most C CTAs
    auto parts = [&](double cap) {
        int k = 1;
        double acc = 0.0;
        for (int v = 0; v < V; ++v) {
            if (acc + cost[v] > cap) {
                ++k;
                acc = 0.0;
            }
            acc += cost[v];
        }
        return k;
    };
    for (int it = 0; it < 60 && hi - lo > 0.5; ++it) {
        const double mid = 0.5 * (lo + hi);
        if (parts(mid) <= C)
            hi = mid;
        else
            lo = mid;
    }
    std::vector<int> cut{0};
    double acc = 0.0;
    for (int v = 0; v < V; ++v) {
        if (acc + cost[v] > hi && v > cut.back()) {
            cut.push_back(v);
            acc = 0.0;
        }
        acc += cost[v];
    }
    cut.push_back(V);
    // exactly C non-empty ranges: split the range with the most panels
    while ((int)cut.size() - 1 < C) {
        int best = 0;
        for (int q = 1; q + 1 < (int)cut.size(); ++q)
            if (cut[q + 1] - cut[q] > cut[best + 1] - cut[best]) best = q;
        cut.insert(cut.begin() + best + 1, (cut[best] + cut[best + 1]) / 2);
    }
    double worst = 0.0;
    for (int q = 0; q < C; ++q) {
        vsplit[q] = cut[q];
        double w = 0.0;
        for (int v = cut[q]; v < cut[q + 1]; ++v) w += cost[v];
        worst = std::max(worst, w);
    }
    vsplit[C] = V;
    return worst;
}

// Dynamic shared memory of a CTA with cpb chunks of rows and KB bases:
// tables, z, rings, row scales, row partials and the inbox of row partials
// pushed by the cluster (C * ceil(R / C) <= R + C floats).
size_t smem_for(int cpb, int KB, int nv, int nw) {
    const size_t R = (size_t)cpb * kChunkRows;
    const int slots = nw == 16 ? Shape<16>::kSlots : Shape<8>::kSlots;
    return (size_t)kTableBytes + kZBytes + (size_t)slots * cpb * 1024 + R * KB * 4 + R * 4 +
           ((R + kMaxCluster + 1) & ~(size_t)1) * 4 + (size_t)nv * sizeof(PanelDesc);
}

// Dynamic shared memory of a stream_kernel CTA with cpb chunks of rows:
// tables, z of two panels, the cluster inbox (C * ceil(R / C) <= R + C floats).
size_t stream_smem(int cpb) {
    return (size_t)kTableBytes + kZBytes + (size_t)((cpb * kChunkRows + kMaxCluster + 1) & ~1) * 4;
}

int stream_items(int cpb) { return cpb <= kStreamWarps ? 1 : cpb <= 2 * kStreamWarps ? 2 : 4; }

// Plan of the streaming kernel (8 warps, two CTAs per SM, up to 4 chunks per
// warp, clusters of up to 16 CTAs).
//  * Independent calls overlap their neighbours: the largest row blocks
//    (fewest table builds per row), C = 2 for matrices of at most 8 row
//    blocks, else 1.
//  * A dependent call is timed alone: latency model of a fixed cost plus,
//    per panel a CTA works through, a table build and its lookups, times
//    the waves; clusters beyond one CTA add a reduction.
Plan make_stream_plan(const fb_weights *W, int batch, int sms, bool independent, int G) {
    Plan pl;
    pl.M_pad = round_up(W->M, kChunkRows);
    pl.Pg = num_panels(W->N);
    pl.nS_pad = W->nS > 0 ? round_up(W->nS, 32) : 0;
    pl.Ps = W->nS > 0 ? num_panels(pl.nS_pad) : 0;
    const std::vector<int> groups = vpanel_groups(W->N, W->K, G == 128, pl.nS_pad, W->nS > 0 ? W->Ks : 0);
    pl.V = (int)groups.size();
    pl.nchunks = pl.M_pad / kChunkRows;
    pl.nwarps = kStreamWarps;
    pl.kind = 1;
    const int max_cpb = 4 * kStreamWarps;
    auto set = [&](int C, int cpb) {
        pl.C = std::min(C, pl.V);
        pl.cpb = std::min(cpb, pl.nchunks);
        pl.RB = ceil_div(pl.nchunks, pl.cpb);
        split_weighted(groups, pl.C, pl.cpb, pl.vsplit);
    };
    if (independent) {
        const int RB = ceil_div(pl.nchunks, max_cpb);
        set(RB <= 8 ? 2 : 1, ceil_div(pl.nchunks, RB));
    } else {
        // One CTA per SM at most (the next call's CTAs take the SMs' other
        // half), minimising the largest CTA's shared-memory work (table
        // builds and lookups, split_weighted) plus a cluster-reduction term.
        // Row blocks of whole chunks per warp (8, 16, 24 or 32 chunks; the
        // whole matrix when it has fewer than 8).
        double best = 1e300;
        set(1, std::min(max_cpb, pl.nchunks));
        for (int cpb = kStreamWarps; cpb <= max_cpb; cpb += kStreamWarps) {
            const int c = std::min(cpb, pl.nchunks);
            const long RB = ceil_div(pl.nchunks, c);
            if (RB > 65535) continue;
            for (int C = 1; C <= std::min(kMaxCluster, pl.V); ++C) {
                const long ctas = (long)C * RB * batch;
                const double waves = std::ceil((double)ctas / sms);
                int vs[kMaxCluster + 1];
                const double work = split_weighted(groups, C, c, vs);
                const double cost = waves * work + (C > 1 ? 1000.0 : 0.0);
                if (cost < best * 0.999) {
                    best = cost;
                    set(C, c);
                }
            }
            if (c == pl.nchunks) break;
        }
    }
    if (const char *ov = getenv("FB_PLAN")) {
        int oc = 0, ocpb = 0;
        if (sscanf(ov, "%d,%d", &oc, &ocpb) == 2 && oc >= 1 && ocpb >= 1)
            set(std::min(oc, kMaxCluster), std::min(ocpb, max_cpb));
    }
    pl.items = stream_items(pl.cpb);
    pl.smem = stream_smem(pl.cpb);
    return pl;
}

// Plan of the batched kernel (16 warps, one CTA per SM): row blocks of up
// to 32 chunks (two per warp), up to 16 tokens per pass, and as many CTAs
// per cluster (up to 16) as fill the SMs once.
size_t batched_smem(int cpb, int tp) {
    return (size_t)2 * kPairTableBytes + 4 * kPanelCols * 4 + (size_t)tp * cpb * kChunkRows * 4;
}

Plan make_batched_plan(const fb_weights *W, int batch, int sms) {
    Plan pl;
    pl.M_pad = round_up(W->M, kChunkRows);
    pl.Pg = num_panels(W->N);
    pl.nS_pad = W->nS > 0 ? round_up(W->nS, 32) : 0;
    pl.Ps = W->nS > 0 ? num_panels(pl.nS_pad) : 0;
    pl.V = pl.Pg * W->K + pl.Ps * (W->nS > 0 ? W->Ks : 0);
    pl.nchunks = pl.M_pad / kChunkRows;
    pl.nwarps = kBatchWarps;
    pl.kind = 2;
    pl.tp = std::min(batch, kMaxTokensPerPass);
    pl.passes = ceil_div(batch, pl.tp);
    const int max_cpb = 2 * kBatchWarps;
    pl.RB = ceil_div(pl.nchunks, max_cpb);
    pl.cpb = ceil_div(pl.nchunks, pl.RB);
    const long blocks = (long)pl.RB * pl.passes;
    int C = blocks >= sms ? 1 : (int)(sms / blocks);
    C = std::max(1, std::min(std::min(C, kMaxCluster), pl.V));
    if (const char *ov = getenv("FB_PLAN")) {
        int oc = 0, ocpb = 0;
        if (sscanf(ov, "%d,%d", &oc, &ocpb) == 2 && oc >= 1 && ocpb >= 1) {
            C = std::min(std::min(oc, kMaxCluster), pl.V);
            pl.cpb = std::min(std::min(ocpb, max_cpb), pl.nchunks);
            pl.RB = ceil_div(pl.nchunks, pl.cpb);
        }
    }
    pl.C = C;
    split_weighted(vpanel_groups(W->N, W->K, 0, pl.nS_pad, W->nS > 0 ? W->Ks : 0), pl.C, pl.cpb, pl.vsplit);
    pl.items = pl.cpb <= kBatchWarps ? 1 : 2;
    pl.smem = batched_smem(pl.cpb, pl.tp);
    return pl;
}

// The launch plan: cluster size C (the split of the V virtual panels over
// the cluster's CTAs) and row block size (cpb chunks of 32 rows).
//  * Calls flagged independent (16-warp CTAs) overlap their neighbours, so
//    the plan that does the least work wins: the largest row blocks (fewest
//    table builds per row), C = 2 for matrices of at most 8 row blocks,
//    else 1.
//  * A dependent call (8-warp CTAs, two per SM) is timed alone: its latency
//    is about a fixed 4 us plus 1.2 us per panel a CTA works through (build,
//    barrier, lookups), times the number of waves; more CTAs per cluster
//    shorten a CTA's panel list.
// Both rules were fitted to timings of this kernel on B200.
Plan make_plan(const fb_weights *W, int batch, int sms, bool independent, bool slots, int G) {
    if (G > 0 || !slots) {
        if (batch > 1) return make_batched_plan(W, batch, sms);
        Plan pl = make_stream_plan(W, batch, sms, independent, G);
        pl.tp = 1;
        pl.passes = 1;
        return pl;
    }
    Plan pl;
    pl.kind = 0;
    pl.items = 2;
    pl.tp = 1;
    pl.passes = batch;
    pl.M_pad = round_up(W->M, kChunkRows);
    pl.Pg = num_panels(W->N);
    pl.nS_pad = W->nS > 0 ? round_up(W->nS, 32) : 0;
    pl.Ps = W->nS > 0 ? num_panels(pl.nS_pad) : 0;
    pl.V = pl.Pg * W->K + pl.Ps * (W->nS > 0 ? W->Ks : 0);
    pl.nchunks = pl.M_pad / kChunkRows;
    const int nw = independent ? 16 : 8, max_cpb = 2 * nw;   // the CTA shape (Shape<NW>)
    pl.nwarps = nw;
    const int KB = W->K + (W->nS > 0 ? W->Ks : 0);
    const int occ_regs = 65536 / (nw * 32 * 128);   // CTAs per SM by registers (128 per thread)
    auto fits = [&](int C, int cpb) {
        int vs[kMaxCluster + 1], nvm;
        split_panels(pl.V, C, vs, &nvm);
        return smem_for(cpb, KB, nvm, nw) <= kMaxDynSmem;
    };
    auto set = [&](int C, int cpb) {
        pl.C = C;
        pl.RB = ceil_div(pl.nchunks, cpb);
        // independent plans balance the row blocks (the same rows, less padding)
        pl.cpb = independent ? ceil_div(pl.nchunks, pl.RB) : cpb;
        int nvm;
        split_panels(pl.V, C, pl.vsplit, &nvm);
    };
    if (independent) {
        int cpb = std::min(max_cpb, pl.nchunks);
        while (cpb > 1 && !fits(2, cpb)) --cpb;
        const int RB = ceil_div(pl.nchunks, cpb);
        set(std::min(pl.V, RB <= 8 ? 2 : 1), cpb);
    } else {
        const double fixed = 4.0, per_panel = 1.2, per_item = 0.1;   // microseconds
        double best = 1e300;
        set(1, std::min(max_cpb, pl.nchunks));
        for (int C = 1; C <= std::min(kMaxSlotCluster, pl.V); ++C) {
            int vs[kMaxCluster + 1], nvm;
            split_panels(pl.V, C, vs, &nvm);
            // whole chunks per warp (uneven splits measured slower on B200), or
            // the whole matrix when it has fewer chunks than warps
            for (int cpb = std::min(nw, pl.nchunks); cpb <= std::min(max_cpb, pl.nchunks);
                 cpb += (pl.nchunks < nw ? max_cpb : nw)) {
                const int RB = ceil_div(pl.nchunks, cpb);
                if (RB > 65535) continue;
                const size_t smem = smem_for(cpb, KB, nvm, nw);
                if (smem > kMaxDynSmem) continue;
                const int occ = std::max(1, std::min(occ_regs, (int)(kSmemPerSM / (smem + kStaticSmem + 1024))));
                const long ctas = (long)C * RB * batch;
                const double waves = std::ceil((double)ctas / ((double)sms * occ));
                const double cost = waves * (fixed + nvm * (per_panel + std::ceil((double)cpb / nw) * per_item));
                if (cost < best * 0.999) {
                    best = cost;
                    set(C, cpb);
                }
            }
        }
    }
    // Tuning aid: FB_PLAN="C,cpb" forces the cluster size and row block
    // (clamped to what the matrix allows); read at each plan construction.
    if (const char *ov = getenv("FB_PLAN")) {
        int oc = 0, ocpb = 0;
        if (sscanf(ov, "%d,%d", &oc, &ocpb) == 2 && oc >= 1 && ocpb >= 1) {
            pl.C = std::min(std::min(oc, kMaxSlotCluster), pl.V);
            pl.cpb = std::min(std::min(ocpb, max_cpb), pl.nchunks);
            int nvm;
            split_panels(pl.V, pl.C, pl.vsplit, &nvm);
            while (pl.cpb > 1 && smem_for(pl.cpb, KB, nvm, nw) > kMaxDynSmem) --pl.cpb;
            pl.RB = ceil_div(pl.nchunks, pl.cpb);
        }
    }
    int nv_max = 0;
    for (int jj = 0; jj < pl.C; ++jj) nv_max = std::max(nv_max, pl.vsplit[jj + 1] - pl.vsplit[jj]);
    pl.smem = smem_for(pl.cpb, KB, nv_max, nw);
    return pl;
}

// Which kernel a call runs: the streaming kernel, except for the test mode
// of the weight-copy waits (only the slot kernel copies weights and waits).
bool use_slots(unsigned flags) {
    (void)flags;
    const char *k = getenv("FB_KERNEL");
    return k && k[0] == 's' && k[1] == 'l';
}

const Plan &cached_plan(const fb_weights *W, int batch, int sms, bool independent, bool slots, int G = 0) {
    struct Entry {
        PlanKey key;
        Plan plan;
    };
    thread_local Entry memo[16];
    thread_local int used = 0, next = 0;
    const PlanKey key{W->M, W->N, W->K, W->g, W->nS, W->nS > 0 ? W->Ks : 0, batch, sms, G, independent, slots};
    for (int i = 0; i < used; ++i)
        if (memo[i].key == key) return memo[i].plan;
    Entry &e = memo[next];
    e.key = key;
    e.plan = make_plan(W, batch, sms, independent, slots, G);
    next = (next + 1) % 16;
    used = std::min(used + 1, 16);
    return e.plan;
}

// Raise the kernel's dynamic shared-memory limit once per kernel and device
// (callers may launch from several host threads: the record is locked).
bool prepare_kernel(KernelFn fn, size_t smem) {
    struct Entry {
        KernelFn fn;
        int dev;
        size_t smem;
    };
    static std::mutex lock;
    static Entry done[64];
    static int n_done = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> guard(lock);
    for (int i = 0; i < n_done; ++i)
        if (done[i].fn == fn && done[i].dev == dev && done[i].smem >= smem) return true;
    const size_t want = std::max<size_t>(smem, 100 * 1024);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)want) != cudaSuccess)
        return false;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) return false;
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

// One launch for n matrices of one format that read the same X (n = 1: a
// plain call).  Y[m] is matrix m's output with row stride ldy[m].
static fb_status launch_gemv(const fb_weights *const *Ws, int n, const void *X, fb_dtype t, int batch, int ldx,
                             float *const *Y, const int *ldy, unsigned flags, void *stream, int G = 0) {
    const fb_weights *W = Ws[0];
    const int es = dtype_size(t);
    if (!X || !es || batch < 1 || batch > kMaxBatch || ldx < W->N || (flags & ~kKnownFlags) ||
        ((flags & FB_GEMV_INDEPENDENT) && !(flags & FB_GEMV_PDL)))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(X, es)) return FB_ERR_MISALIGNED;
    int M_max = 0;
    for (int m = 0; m < n; ++m) {
        if (!Y[m] || ldy[m] < Ws[m]->M) return FB_ERR_INVALID_VALUE;
        if (!aligned(Y[m], 4)) return FB_ERR_MISALIGNED;
        M_max = std::max(M_max, Ws[m]->M);
    }
    // the plan of the largest matrix (the format, hence the panels, is shared)
    fb_weights Wp = *W;
    Wp.M = M_max;
    const Plan &pl = cached_plan(&Wp, batch, sm_count(), (flags & FB_GEMV_INDEPENDENT) != 0, use_slots(flags), G);
    const KernelFn fn = pl.kind == 0 ? pick_kernel(t, pl.nwarps)
                        : pl.kind == 1 ? pick_stream(t, pl.items) : pick_batched(t, pl.items);
    if (!prepare_kernel(fn, pl.smem)) return FB_ERR_CUDA;

    GemvArgs a;
    a.group = n;
    a.rb_base = 0;
    a.rb_start[0] = 0;
    for (int m = 0; m < kMaxGroup; ++m) {
        GemvArgs::Mat &mt = a.mats[m];
        const fb_weights *Wm = Ws[std::min(m, n - 1)];
        mt.planes = (const uint8_t *)Wm->planes;
        mt.alpha_r = Wm->alpha_r;
        mt.alpha_c = Wm->alpha_c;
        mt.s_planes = (const uint8_t *)Wm->s_planes;
        mt.s_alpha_r = Wm->s_alpha_r;
        mt.s_alpha_c = Wm->s_alpha_c;
        mt.s_idx = Wm->s_idx;
        mt.y = Y[std::min(m, n - 1)];
        mt.M = Wm->M;
        mt.M_pad = round_up(Wm->M, kChunkRows);
        mt.nchunks = mt.M_pad / kChunkRows;
        mt.pad = 0;
        if (m < n) a.rb_start[m + 1] = a.rb_start[m] + ceil_div(mt.nchunks, pl.cpb);
    }
    for (int m = n; m < kMaxGroup; ++m) a.rb_start[m + 1] = a.rb_start[n];
    const int rows_of_blocks = a.rb_start[n];
    if (rows_of_blocks > 65535) return FB_ERR_UNSUPPORTED;
    a.planes = a.mats[0].planes;
    a.alpha_r = a.mats[0].alpha_r;
    a.alpha_c = a.mats[0].alpha_c;
    a.s_planes = a.mats[0].s_planes;
    a.s_alpha_r = a.mats[0].s_alpha_r;
    a.s_alpha_c = a.mats[0].s_alpha_c;
    a.s_idx = a.mats[0].s_idx;
    a.x = X;
    a.y = Y[0];
    a.M = W->M;
    a.M_pad = a.mats[0].M_pad;
    a.N = W->N;
    a.K = W->K;
    a.nS = W->nS;
    a.nS_pad = pl.nS_pad;
    a.Ks = W->nS > 0 ? W->Ks : 0;
    a.Pg = pl.Pg;
    a.Ps = pl.Ps;
    a.nchunks = a.mats[0].nchunks;
    a.cpb = pl.cpb;
    a.ldx = ldx;
    a.ldy = ldy[0];
    a.flags = flags;
    a.C = pl.C;
    a.batch = batch;
    a.tp = pl.tp;
    a.G = G;
    a.ngr = G > 0 ? W->N / G : 1;
    a.KR = W->K * a.ngr;
    a.hsplit = G == 128;
    std::copy(pl.vsplit, pl.vsplit + kMaxCluster + 1, a.vsplit);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.C, rows_of_blocks, pl.passes);
    cfg.blockDim = dim3(pl.nwarps * 32);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = as_stream(stream);
    cudaLaunchAttribute attr[3];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // a cluster's CTAs on different SMs: two CTAs of one call sharing an SM
    // would each run at half speed, and the cluster waits for its slowest
    attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[1].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
    int na = 2;
    if (flags & FB_GEMV_PDL) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return status_of(cudaLaunchKernelEx(&cfg, fn, a));
}

extern "C" fb_status fb_gemv_batched(const fb_weights *W, const void *X, fb_dtype t, int batch, int ldx,
                                     float *Y, int ldy, void *ws, size_t ws_bytes, unsigned flags,
                                     void *stream) {
    (void)ws;
    (void)ws_bytes;
    const fb_status st = check_weights(W);
    if (st != FB_OK) return st;
    const fb_weights *Ws[1] = {W};
    float *Ys[1] = {Y};
    const int ldys[1] = {ldy};
    return launch_gemv(Ws, 1, X, t, batch, ldx, Ys, ldys, flags, stream);
}

extern "C" fb_status fb_gemv_grouped(const fb_weights *const *W, int n, const void *x, fb_dtype t, float *const *y,
                                     unsigned flags, void *stream) {
    if (!W || !y || n < 1 || n > kMaxGroup) return FB_ERR_INVALID_VALUE;
    int ldy[kMaxGroup];
    for (int m = 0; m < n; ++m) {
        const fb_status st = check_weights(W[m]);
        if (st != FB_OK) return st;
        const fb_weights *A = W[0], *B = W[m];
        const int ksA = A->nS > 0 ? A->Ks : 0, ksB = B->nS > 0 ? B->Ks : 0;
        if (B->N != A->N || B->K != A->K || B->g != A->g || B->nS != A->nS || ksB != ksA)
            return FB_ERR_INVALID_VALUE;   // not one format
        ldy[m] = B->M;
    }
    return launch_gemv(W, n, x, t, 1, W[0]->N, y, ldy, flags, stream);
}

extern "C" fb_status fb_gemv_launch_plan(const fb_weights *W, int batch, unsigned flags, int sms, int *out) {
    if (check_weights(W) != FB_OK || batch < 1 || batch > kMaxBatch || sms < 1 || !out || (flags & ~kKnownFlags))
        return FB_ERR_INVALID_VALUE;
    const Plan &pl = cached_plan(W, batch, sms, (flags & FB_GEMV_INDEPENDENT) != 0, use_slots(flags));
    out[0] = pl.C;
    out[1] = pl.cpb;
    out[2] = pl.RB;
    out[3] = pl.nwarps;
    out[4] = (int)pl.smem;
    out[5] = pl.V;
    return FB_OK;
}

extern "C" fb_status fb_gemv(const fb_weights *W, const void *x, fb_dtype t, float *y, void *ws,
                             size_t ws_bytes, unsigned flags, void *stream) {
    if (!W) return FB_ERR_INVALID_VALUE;
    return fb_gemv_batched(W, x, t, 1, W->N, y, W->M, ws, ws_bytes, flags, stream);
}

extern "C" fb_status fb_gemv_group_scales(const fb_weights *W, int G, const void *x, fb_dtype t, float *y,
                                          unsigned flags, void *stream) {
    const fb_status st = check_weights(W);
    if (st != FB_OK) return st;
    if (!(G == 128 || G == W->N || (G > 0 && G % kPanelCols == 0)) || W->N % G != 0) return FB_ERR_INVALID_VALUE;
    const fb_weights *Ws[1] = {W};
    float *Ys[1] = {y};
    const int ldys[1] = {W->M};
    return launch_gemv(Ws, 1, x, t, 1, W->N, Ys, ldys, flags, stream, G);
}

extern "C" fb_status fb_device_errors(unsigned int *flags, int clear) {
    if (!flags) return FB_ERR_INVALID_VALUE;
    if (cudaDeviceSynchronize() != cudaSuccess) return FB_ERR_CUDA;
    if (cudaMemcpyFromSymbol(flags, g_error_flags, sizeof(unsigned int)) != cudaSuccess) return FB_ERR_CUDA;
    if (clear) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_error_flags, &zero, sizeof(unsigned int)) != cudaSuccess) return FB_ERR_CUDA;
    }
    return FB_OK;
}
