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
// chunks; CTA j of the cluster takes a contiguous slice of the V virtual
// panels (balanced by their lookup work), so the cluster covers every column
// of its rows.
//
// stream_kernel (batch 1; 8 warps, three CTAs per SM for calls flagged
// independent and two otherwise, or 16 warps, one):
//   1. the words of the CTA's first panel (two for warps of one or two
//      items) are loaded straight into registers (each lane its rows' bytes,
//      128-bit loads), with the row scales; for calls that depend on the
//      previous kernel this, and an L2 prefetch of the next panels, happens
//      before the programmatic-launch wait, and x is read after it;
//   2. per panel, the CTA builds the panel's byte tables in shared memory
//      (LUT-BSF: z = alpha_c * x, salient panels reading x[s_idx[t]] -- the
//      virtual columnar mapping -- and for each group of 8 columns the 256
//      sums sum_t (bit t of b ? +z_t : -z_t), each the sum of the two 4-column
//      tables of its nibbles), double-buffered, one CTA barrier per panel;
//      right after an item's lookups its registers take the same item of a
//      later panel;
//   3. each lane walks its row's bytes: one `prmt` merges a weight byte and
//      the lane's column offset into a table address, one shared load fetches
//      the partial sum, packed fp32x2 adds accumulate (a gather-add, no tensor
//      cores); each item's sum is scaled by alpha_r once (alpha_r applied in
//      the reduction) and added to the row's partial;
//   4. each row partial is sent to the cluster CTA that owns the row as an
//      asynchronous remote store completing on the owner's barrier; the
//      owner waits (bounded) for all of them and sums its C slots in rank
//      order.  No workspace, no atomics; deterministic.
// batched_kernel (several tokens): the same, with each panel's words applied
// to every token of a pass in turn (one weight pass per pass of tokens).
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
constexpr int kMaxGroup = 4;            // matrices in one grouped call
constexpr size_t kMaxDynSmem = 225 * 1024;   // dynamic shared memory per CTA
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

// Column staging in two phases, so no thread waits on the salient column
// index while it stages: stage_column issues the loads of column c's scale
// and -- for a global column -- of its x; for a salient column it loads the
// index s_idx (xi = kPendingIndex, the raw index in x), and resolve_column,
// one panel later, turns the index into the x column and issues that load.
constexpr int kPendingIndex = -2;

struct Staged {
    float ac;     // alpha_c of the column (0: none)
    uint32_t x;   // stored bits of x[xi]; or the raw salient index while xi == kPendingIndex
    int xi;       // column of x, -1 (none) or kPendingIndex
};

template <int XT, bool kDup>
__device__ __forceinline__ void stage_column(const GemvArgs &a, const PanelDesc &d, int c, size_t xoff, bool read_x,
                                             Staged &t) {
    t.ac = 0.0f;
    t.xi = -1;
    t.x = 0;
    const int w = desc_bp(d) * 8;
    if (c >= w) {
        if (!kDup || c >= (kPanelCols / w) * w) return;
        c -= (c / w) * w;
    }
    const int half = desc_half(d);
    if (half && (c >> 7) != half - 1) return;
    const int col = d.col0 + c;
    if (!desc_sal(d)) {
        t.xi = col;
        t.ac = d.ac ? __ldg(d.ac + col) : 1.0f;
        if (read_x) t.x = load_x_bits<XT>(a.x, xoff + col);
    } else if (col < a.nS) {
        t.ac = __ldg(d.ac + col);
        t.x = __ldg(a.s_idx + col);
        t.xi = kPendingIndex;
    }
}

template <int XT>
__device__ __forceinline__ void resolve_column(const GemvArgs &a, size_t xoff, Staged &t) {
    if (t.xi != kPendingIndex) return;
    const uint32_t jx = t.x;
    t.xi = jx < (uint32_t)a.N ? (int)jx : -1;   // an invalid index contributes 0
    t.x = t.xi >= 0 ? load_x_bits<XT>(a.x, xoff + t.xi) : 0u;
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

// Where column t of a panel keeps its z in the z buffer: the low four
// columns of every 8-column group first (group q at 4q), then the high four
// (at 128 + 4q), so that lane q reads its group as two 16-byte words at
// consecutive addresses across the warp (4 wavefronts each, not 8).
__device__ __forceinline__ int z_slot(int t) { return ((t & 4) ? kPanelCols / 2 : 0) + 4 * (t >> 3) + (t & 3); }

// LUT-BSF for one virtual panel, built by the whole CTA: lane q builds byte
// group q (columns 8q .. 8q+7, their z at z_slot in zp), warp w its entries
// b = 32w .. 32w+31:
// entry b = T_lo[b & 15] + T_hi[b >> 4], where T_lo and T_hi are the 16-entry
// tables of the group's low and high 4 columns, each (+-z0 +- z1) + (+-z2 +-
// z3).  Columns past a narrow panel's width have z = 0, so their entries are
// 0.  T points at the buffer (entry b of group q at T[b*64 + q]).  Each of
// the NW warps writes 256 / NW consecutive entries b of every group.
template <int NW>
__device__ __forceinline__ void build_byte_table(const float *zp, float *T, int warp, int lane) {
    constexpr int kHi = 16 / NW;   // high-nibble values per warp: entries b = 16*kHi*warp ...
    const float4 za = *reinterpret_cast<const float4 *>(zp + 4 * lane);
    const float4 zb = *reinterpret_cast<const float4 *>(zp + kPanelCols / 2 + 4 * lane);
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

// Set (bit 0) when a CTA gave up waiting for its cluster's row partials;
// the rows it owns are then written as NaN.  Read and cleared by
// fb_device_errors.
__device__ unsigned int g_error_flags;

// One lane's words of one item: position u in byte u % 4 of w[u / 4].
struct Words {
    uint32_t w[8];
};
// Shared memory of the byte tables (two interleaved buffers) and of the z
// values of two panels.
constexpr int kTableBytes = 65536;
constexpr int kZBytes = 2 * kPanelCols * 4;
// ---- The streaming kernel: weights straight into registers --------------
//
// The packed weights are not staged in shared memory: each lane loads its
// rows' words of a later panel with 128-bit loads into registers right
// after it has looked up the current ones, so a weight byte costs
// shared-memory bandwidth only for its table lookup.  8 warps per CTA and
// about 70 KB of shared memory let two or three CTAs share an SM, so one
// CTA's prologue, barriers and reduction overlap the others' lookups.  For
// calls that depend on the previous kernel the first panel's words (two
// panels' for warps of one or two items) and an L2 prefetch of the next
// panels are requested before the programmatic-launch wait.

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

// CTAs per SM the kernel is compiled for (its register budget): three for
// calls flagged independent with up to four items per warp (80 registers,
// 24 warps per SM: the overlapped calls' latency is hidden by more warps),
// two otherwise (128 registers: a call that waits for its predecessor is
// bound by each CTA's own critical path, and keeps an SM slot free for the
// next call's CTAs).
template <int XT, int NW, int I, int kBlocks>
__global__ void __launch_bounds__(NW * 32, kBlocks) stream_kernel(const __grid_constant__ GemvArgs args) {
    static_assert(NW == 8 || NW == 16, "8 warps (two or three CTAs per SM) or 16 (one)");
    constexpr bool kAllStage = NW * 32 == kPanelCols;   // every thread stages a column
    extern __shared__ __align__(128) float smem_f[];
    __shared__ __align__(16) GemvArgs s_args;
    __shared__ __align__(16) PanelDesc s_ring[kDescRing];
    __shared__ __align__(8) unsigned long long s_inbox_bar;   // the cluster's row partials have landed
    // The next call in the stream may launch at once: it reads nothing this
    // kernel writes before its own programmatic-launch wait, and a call
    // flagged independent completes only after this one.
    griddep_launch_dependents();
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

    // ---- 1. before the wait: the first D panels' words and row scales, the
    // column sources of panel 0 (and its x when independent) ---------------
    // A ring of D register sets (two for warps of one or two items, whose
    // panels are short; one for more): right after an item's lookups in panel
    // v, its registers take the same item of panel v + D, so each load has D
    // panels' time to land, and a CTA of one or two panels has all its words
    // requested before the wait.  (Four sets for one item lengthened the
    // dependent chain of a 7B-shaped layer, whose calls alternate between
    // kernels, by 7%: the four-panel loop body is twice the code.)
    constexpr int D = I <= 2 ? 2 : 1;
    uint32_t w[D][I][8];
    float rar[D][I];
    auto load_item = [&](auto slotc, int i, const PanelDesc &d) {
        constexpr int sl = decltype(slotc)::value;
        const int Bp = desc_bp(d);
        const size_t blk = 32u * (unsigned)Bp;
        const int cl = warp + NW * i;
        const int row = (c_first + cl) * kChunkRows + lane;
        rar[sl][i] = cl < nvalid && row < a.M ? __ldg(row_scales(a, d.kb) + row) : 0.0f;
        if (cl < nvalid) {
            const uint8_t *p = d.pl + blk * (size_t)(c_first + cl);
            if (Bp == 32) {
                const uint4 x0 = ldg_stream(p + 16 * lane), x1 = ldg_stream(p + 512 + 16 * lane);
                w[sl][i][0] = x0.x; w[sl][i][1] = x0.y; w[sl][i][2] = x0.z; w[sl][i][3] = x0.w;
                w[sl][i][4] = x1.x; w[sl][i][5] = x1.y; w[sl][i][6] = x1.z; w[sl][i][7] = x1.w;
            } else {
                const Words r = load_item_narrow(p, Bp, lane);
#pragma unroll
                for (int m = 0; m < 8; ++m) w[sl][i][m] = r.w[m];
            }
        }
    };
    auto load_panel = [&](auto slotc, const PanelDesc &d) {
#pragma unroll
        for (int i = 0; i < I; ++i) load_item(slotc, i, d);
    };
    if (tid < kDescRing - 4 && tid < n_v) s_ring[tid] = panel_desc(a, vb + tid);
    Staged st[2] = {{0.0f, 0u, -1}, {0.0f, 0u, -1}};
    auto stage = [&](Staged &t, const PanelDesc &d, bool read_x) {
        if (kAllStage || tid < kPanelCols) stage_column<XT, true>(a, d, tid, xoff, read_x, t);
    };
    auto resolve = [&](Staged &t) { resolve_column<XT>(a, xoff, t); };
    auto z_of = [&](const Staged &t) { return t.xi >= 0 ? __fmul_rn(t.ac, x_value<XT>(t.x)) : 0.0f; };
    PanelDesc d1;
    if (n_v > 0) {
        const PanelDesc d0 = panel_desc(a, vb);
        load_panel(std::integral_constant<int, 0>{}, d0);
        stage(st[0], d0, independent);
    }
    if (n_v > 1) d1 = panel_desc(a, vb + 1);
    if (D > 1 && n_v > 1) load_panel(std::integral_constant<int, D - 1>{}, d1);
    if (!independent) {
        // the rest of the slice into L2 while the previous kernel finishes
        if (tid == 0) {
            for (int v = D; v < min(n_v, 8); ++v) {
                const PanelDesc d = panel_desc(a, vb + v);
                const uint32_t blk = 32u * (uint32_t)desc_bp(d);
                prefetch_l2(d.pl + (size_t)blk * c_first, blk * (uint32_t)nvalid);
            }
        }
        griddep_wait();
        if (st[0].xi >= 0) st[0].x = load_x_bits<XT>(a.x, xoff + st[0].xi);
    }
    if (n_v > 1) stage(st[1], d1, true);   // x of panel 1 in flight with panel 0's
    resolve(st[0]);
    if (n_v > 1) resolve(st[1]);
    if (kAllStage || tid < kPanelCols) zbuf[z_slot(tid)] = z_of(st[0]);
    __syncthreads();   // z of panel 0 and the first descriptors written
    if (n_v > 2) stage(st[0], s_ring[2], true);

    uint32_t off_full[8];
    full_offsets(lane, off_full);

    float racc[I];
#pragma unroll
    for (int i = 0; i < I; ++i) racc[i] = 0.0f;

    // ---- 2. per panel: tables, then this warp's items ----------------------
    // (table buffer buf = vi % 2, register set slotc = vi % D)
    auto panel = [&](auto bufc, auto slotc, int vi) {
        constexpr int buf = decltype(bufc)::value;
        constexpr int sl = decltype(slotc)::value;
        const int Bp = desc_bp(s_ring[vi % kDescRing]);
        float *tb = tables + 32 * buf;
        build_byte_table<NW>(zbuf + buf * kPanelCols, tb, warp, lane);
        if (vi + 1 < n_v && (kAllStage || tid < kPanelCols))
            zbuf[(buf ^ 1) * kPanelCols + z_slot(tid)] = z_of(st[buf ^ 1]);
        if (vi + 3 < n_v) stage(st[buf ^ 1], s_ring[(vi + 3) % kDescRing], true);
        if (vi + 2 < n_v) resolve(st[buf]);   // panel vi + 2, staged one panel ago
        if (tid == 0 && vi + 4 < n_v) s_ring[(vi + 4) % kDescRing] = panel_desc(a, vb + vi + 4);
        __syncthreads();   // tables of panel vi complete; every warp done with panel vi - 1
        const bool more = vi + D < n_v;
        const PanelDesc &nd = s_ring[(vi + D) % kDescRing];   // panel vi + D (its items load here)
        if (Bp == 32) {
#pragma unroll
            for (int i = 0; i < I; i += 2) {
                const int c0 = warp + NW * i;
                if (i + 1 < I && c0 + NW < nvalid) {
                    float s0, s1;
                    lookup_rows2(w[sl][i], w[sl][i + 1], off_full, tb, s0, s1);
                    racc[i] = __fadd_rn(racc[i], __fmul_rn(rar[sl][i], s0));
                    racc[i + 1] = __fadd_rn(racc[i + 1], __fmul_rn(rar[sl][i + 1], s1));
                } else if (c0 < nvalid) {
                    racc[i] = __fadd_rn(racc[i], __fmul_rn(rar[sl][i], lookup_row(w[sl][i], off_full, tb)));
                }
                if (more) {
                    load_item(slotc, i, nd);
                    if (i + 1 < I) load_item(slotc, i + 1, nd);
                }
            }
        } else {
            const Offsets o = narrow_offsets_dup(lane, Bp);
#pragma unroll
            for (int i = 0; i < I; ++i) {
                if (warp + NW * i < nvalid)
                    racc[i] = __fadd_rn(racc[i],
                                        __fmul_rn(rar[sl][i], lookup_row_narrow(w[sl][i], o.w, tb, Bp >> 2)));
                if (more) load_item(slotc, i, nd);
            }
        }
    };
    using C0 = std::integral_constant<int, 0>;
    using C1 = std::integral_constant<int, 1>;
    using S1 = std::integral_constant<int, D - 1>;
#pragma unroll 1
    for (int vi = 0; vi < n_v; vi += 2) {   // panels vi, vi + 1: buffers 0 1, register sets vi % D
        panel(C0{}, C0{}, vi);
        if (vi + 1 < n_v) panel(C1{}, S1{}, vi + 1);
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
    // complete only after the previous kernel: one CTA waiting is enough (the
    // grid completes when its last CTA exits), and the others free their SM
    // slots for the calls that follow
    if (independent && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) griddep_wait();
}

// ---- The batched kernel: one weight pass for the tokens of a pass -------
//
// Several activation vectors share each weight word: a CTA loads a panel's
// words for its rows into registers once (stream_kernel's two register sets,
// the panel after next loading while the current one is used) and applies
// them to every token of its pass in turn.  Each token is one step of
// stream_kernel's panel loop -- z, the 256-entry byte tables, the lookups --
// with the tables double-buffered across consecutive steps; a pass holds an
// even number of tokens, so a step's buffer is its token's parity (a
// compile-time constant, as in stream_kernel).  Per token, every sum is
// formed in exactly stream_kernel's order; the per-token row partials live
// in shared memory.
//
// Shared memory: tables (two interleaved buffers, 64 KB; after the last
// lookups the same bytes receive the cluster's row partials) | z of two
// steps | row partials [tp][R].  8 warps; with 8 tokens per pass two CTAs
// share an SM (128 registers); with 2 tokens per pass, three (kBlocks = 3:
// 80 registers, up to four items per warp).
constexpr int kBatchWarps = 8;
constexpr int kMaxTokensPerPass = 16;

template <int XT, int I, int kBlocks>
__global__ void __launch_bounds__(kBatchWarps * 32, kBlocks) batched_kernel(const __grid_constant__ GemvArgs args) {
    constexpr int NW = kBatchWarps, NT = NW * 32;
    extern __shared__ __align__(128) float smem_f[];
    __shared__ __align__(16) GemvArgs s_args;
    __shared__ __align__(16) PanelDesc s_ring[kDescRing];
    griddep_launch_dependents();   // (as in stream_kernel)
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
    const int S = n_v * TP;   // steps (panel, token), token fastest

    float *tables = smem_f;
    float *zbuf = smem_f + kTableBytes / 4;
    float *accs = zbuf + kZBytes / 4;   // [TP][R]
    float *inbox = tables;              // after the last lookups

    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

    for (int i = tid; i < TP * R; i += NT) accs[i] = 0.0f;
    if (tid < kDescRing - 4 && tid < n_v) s_ring[tid] = panel_desc(a, vb + tid);

    // One weight register set, as in stream_kernel: an item's registers take
    // the next panel's words right after the pass's last token used them.
    uint32_t w[I][8];
    float rar[I];
    auto load_item = [&](int i, const PanelDesc &d) {
        const int Bp = desc_bp(d);
        const size_t blk = 32u * (unsigned)Bp;
        const int cl = warp + NW * i;
        const int row = (c_first + cl) * kChunkRows + lane;
        rar[i] = cl < nvalid && row < a.M ? __ldg(row_scales(a, d.kb) + row) : 0.0f;
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
    };
    Staged st[2] = {{0.0f, 0u, -1}, {0.0f, 0u, -1}};
    int st_tok[2] = {0, 0};   // the token each staged set belongs to
    // column tid of a step's panel, for token tok of the pass (none past nt)
    auto stage = [&](int q, const PanelDesc &d, int tok, bool read_x) {
        st_tok[q] = tok;
        if (tok >= nt) {
            st[q].ac = 0.0f;
            st[q].x = 0;
            st[q].xi = -1;
            return;
        }
        stage_column<XT, true>(a, d, tid, (size_t)(t_base + tok) * a.ldx, read_x, st[q]);
    };
    auto resolve = [&](int q) { resolve_column<XT>(a, (size_t)(t_base + st_tok[q]) * a.ldx, st[q]); };
    auto z_of = [&](const Staged &t) { return t.xi >= 0 ? __fmul_rn(t.ac, x_value<XT>(t.x)) : 0.0f; };

    PanelDesc d0, d1;
    if (n_v > 0) {
        d0 = panel_desc(a, vb);
#pragma unroll
        for (int i = 0; i < I; ++i) load_item(i, d0);
        stage(0, d0, 0, independent);
    }
    if (n_v > 1) d1 = panel_desc(a, vb + 1);
    if (!independent) {
        griddep_wait();
        if (st[0].xi >= 0) st[0].x = load_x_bits<XT>(a.x, (size_t)t_base * a.ldx + st[0].xi);
    }
    if (S > 1) stage(1, d0, 1, true);   // step 1: panel 0 (a pass holds at least two tokens)
    resolve(0);
    if (S > 1) resolve(1);
    zbuf[z_slot(tid)] = z_of(st[0]);
    __syncthreads();   // z of step 0, the first descriptors and the zeroed partials written
    if (S > 2) stage(0, TP > 2 ? d0 : d1, 2 % TP, true);

    uint32_t off_full[8];
    full_offsets(lane, off_full);

    // One step: token tok of panel vi, tables in buffer `buf` (= tok & 1);
    // the pass's last step reloads each item with the next panel's words.
    auto step = [&](auto bufc, int vi, int tok) {
        constexpr int buf = decltype(bufc)::value;
        const int s2 = vi * TP + tok;
        const int Bp = desc_bp(s_ring[vi % kDescRing]);
        float *tb = tables + 32 * buf;
        if (tok < nt) build_byte_table<NW>(zbuf + buf * kPanelCols, tb, warp, lane);
        if (s2 + 1 < S) zbuf[(buf ^ 1) * kPanelCols + z_slot(tid)] = z_of(st[buf ^ 1]);
        if (s2 + 3 < S) {
            const int s3 = s2 + 3, v3 = s3 / TP;
            stage(buf ^ 1, s_ring[v3 % kDescRing], s3 - v3 * TP, true);
        }
        if (s2 + 2 < S) resolve(buf);   // step s2 + 2, staged one step ago
        if (tid == 0 && tok == 0 && vi + 4 < n_v) s_ring[(vi + 4) % kDescRing] = panel_desc(a, vb + vi + 4);
        __syncthreads();   // tables of this step complete; every warp done with the previous step
        // the pass's last token with lookups: after it, the items reload
        const bool reload = tok == min(TP, nt) - 1 && vi + 1 < n_v;
        const PanelDesc &nd = s_ring[(vi + 1) % kDescRing];
        if (tok >= nt) return;
        float *acc_t = accs + tok * R;
        if (Bp == 32) {
#pragma unroll
            for (int i = 0; i < I; i += 2) {
                const int c0 = warp + NW * i;
                if (i + 1 < I && c0 + NW < nvalid) {
                    float s0, s1;
                    lookup_rows2(w[i], w[i + 1], off_full, tb, s0, s1);
                    float *p0 = acc_t + c0 * kChunkRows + lane;
                    *p0 = __fadd_rn(*p0, __fmul_rn(rar[i], s0));
                    float *p1 = p0 + NW * kChunkRows;
                    *p1 = __fadd_rn(*p1, __fmul_rn(rar[i + 1], s1));
                } else if (c0 < nvalid) {
                    float *p0 = acc_t + c0 * kChunkRows + lane;
                    *p0 = __fadd_rn(*p0, __fmul_rn(rar[i], lookup_row(w[i], off_full, tb)));
                }
                if (reload) {
                    load_item(i, nd);
                    if (i + 1 < I) load_item(i + 1, nd);
                }
            }
        } else {
            const Offsets o = narrow_offsets_dup(lane, Bp);
#pragma unroll
            for (int i = 0; i < I; ++i) {
                const int c0 = warp + NW * i;
                if (c0 < nvalid) {
                    float *p0 = acc_t + c0 * kChunkRows + lane;
                    *p0 = __fadd_rn(*p0, __fmul_rn(rar[i], lookup_row_narrow(w[i], o.w, tb, Bp >> 2)));
                }
                if (reload) load_item(i, nd);
            }
        }
    };
#pragma unroll 1
    for (int vi = 0; vi < n_v; ++vi) {
#pragma unroll 1
        for (int tok = 0; tok < TP; tok += 2) {
            step(std::integral_constant<int, 0>{}, vi, tok);
            step(std::integral_constant<int, 1>{}, vi, tok + 1);
        }
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
    if (independent && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) griddep_wait();   // (as stream_kernel)
}

using KernelFn = void (*)(GemvArgs);

template <int I, int B = 2>
KernelFn pick_batched_xt(fb_dtype t) {
    return t == FB_F32 ? batched_kernel<FB_F32, I, B> : t == FB_F16 ? batched_kernel<FB_F16, I, B>
                                                                    : batched_kernel<FB_BF16, I, B>;
}
// The batched kernel for `items` chunks per warp; `three`: the variant with
// three CTAs per SM (up to four items).
KernelFn pick_batched(fb_dtype t, int items, bool three) {
    if (three && items <= 4)
        return items == 1 ? pick_batched_xt<1, 3>(t) : items == 2 ? pick_batched_xt<2, 3>(t)
                                                                   : pick_batched_xt<4, 3>(t);
    return items == 1 ? pick_batched_xt<1>(t) : items == 2 ? pick_batched_xt<2>(t)
                      : items == 4 ? pick_batched_xt<4>(t) : pick_batched_xt<8>(t);
}

template <int NW, int I, int B = 16 / NW>
KernelFn pick_stream_xt(fb_dtype t) {
    return t == FB_F32 ? stream_kernel<FB_F32, NW, I, B> : t == FB_F16 ? stream_kernel<FB_F16, NW, I, B>
                                                                       : stream_kernel<FB_BF16, NW, I, B>;
}
// The streaming kernel for nw warps and `items` chunks per warp; `three`:
// the variant with three CTAs per SM (independent calls, up to four items).
KernelFn pick_stream(fb_dtype t, int nw, int items, bool three) {
    if (nw == 16) return items == 1 ? pick_stream_xt<16, 1>(t) : items == 2 ? pick_stream_xt<16, 2>(t)
                                                                             : pick_stream_xt<16, 4>(t);
    if (three && items <= 4)
        return items == 1 ? pick_stream_xt<8, 1, 3>(t) : items == 2 ? pick_stream_xt<8, 2, 3>(t)
                                                                    : pick_stream_xt<8, 4, 3>(t);
    return items == 1 ? pick_stream_xt<8, 1>(t) : items == 2 ? pick_stream_xt<8, 2>(t)
                      : items == 4 ? pick_stream_xt<8, 4>(t) : pick_stream_xt<8, 8>(t);
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
    int kind;    // 1: stream_kernel; 2: batched_kernel
    int items;   // stream / batched kernel: chunks per warp per panel
    int tp, passes;   // batched kernel: tokens per pass, passes (grid.z)
    int three = 0;    // batched kernel: the variant with three CTAs per SM
    int vsplit[kMaxCluster + 1];
    size_t smem;
};

struct PlanKey {
    int M, N, K, g, nS, Ks, batch, sms, G;
    bool independent;
    int rows[kMaxGroup];   // a grouped call: every matrix's M (0 past the last)
    bool operator==(const PlanKey &o) const {
        return M == o.M && N == o.N && K == o.K && g == o.g && nS == o.nS && Ks == o.Ks && batch == o.batch &&
               sms == o.sms && G == o.G && independent == o.independent &&
               std::equal(rows, rows + kMaxGroup, o.rows);
    }
};

// The matrices of one launch (a grouped call's row blocks follow one another
// in the grid): their row counts.
struct Group {
    int n = 1;
    int M[kMaxGroup] = {0, 0, 0, 0};
};

// Row blocks of a launch whose blocks hold cpb chunks of 32 rows.
long group_row_blocks(const Group &grp, int cpb) {
    long rb = 0;
    for (int m = 0; m < grp.n; ++m) rb += ceil_div(round_up(grp.M[m], kChunkRows) / kChunkRows, cpb);
    return rb;
}

// Clusters of C stream_kernel CTAs that can be resident at once with two
// CTAs per SM.  A cluster stays within one GPC, so this is less than 2 * sms
// / C; the table is cudaOccupancyMaxActiveClusters on B200 (148 SMs) for
// such a kernel, scaled for other SM counts.
int cluster_capacity(int sms, int C) {
    static const int k148[kMaxCluster + 1] = {0, 296, 148, 93, 71, 56, 45, 37, 33, 30, 26, 21, 21, 17, 14, 14, 14};
    return std::max(1, (int)((long)k148[std::min(std::max(C, 1), kMaxCluster)] * sms / 148));
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

// Dynamic shared memory of a stream_kernel CTA with cpb chunks of rows:
// tables, z of two panels, the cluster inbox (C * ceil(R / C) <= R + C floats).
size_t stream_smem(int cpb) {
    return (size_t)kTableBytes + kZBytes + (size_t)((cpb * kChunkRows + kMaxCluster + 1) & ~1) * 4;
}

int stream_items(int cpb, int nw = kStreamWarps) { return cpb <= nw ? 1 : cpb <= 2 * nw ? 2 : cpb <= 4 * nw ? 4 : 8; }

// Plan of the streaming kernel (8 warps, up to 4 chunks per warp -- 8 for
// the largest independent calls and with the tuning override -- and
// clusters of up to 16 CTAs).
//  * Independent calls overlap their neighbours: row blocks of 32 chunks
//    (few table builds per row; 64 from 64 MiB of packed planes), small
//    clusters (for at most 4 row blocks one CTA per ~24 virtual panels,
//    1 up to 40; 2 for at most 8 row blocks; else 1).
//  * A call that waits for its predecessor: the plan of least modelled
//    latency (per panel a CTA works through, a fixed cost and a cost per
//    chunk of rows; times the waves of clusters that fit at two CTAs per
//    SM; plus a cost per CTA of a cluster), row blocks counted over the
//    whole launch of a grouped call.
Plan make_stream_plan(const fb_weights *W, int batch, int sms, bool independent, int G, const Group &grp) {
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
    const int max_cpb = 4 * kStreamWarps;   // default plans: up to 4 items per warp
    auto set = [&](int C, int cpb) {
        pl.C = std::max(1, std::min(std::min(C, pl.V), kMaxCluster));   // (vsplit holds kMaxCluster + 1 cuts)
        pl.cpb = std::min(cpb, pl.nchunks);
        pl.RB = ceil_div(pl.nchunks, pl.cpb);
        split_weighted(groups, pl.C, pl.cpb, pl.vsplit);
    };
    if (independent) {
        // Matrices of at least 64 MiB of packed planes (65536 items): row
        // blocks of 64 chunks (eight per warp) in clusters of 2 -- the
        // fewest table builds per row.  Smaller ones: row blocks of up to 32
        // chunks; matrices of at most 4 row blocks take C = 1 up to 40
        // virtual panels (4096^2: no cluster reduction; 1.377 -> 1.365 us,
        // the 7B-shaped step 0.643 -> 0.613 ms) and about 24 panels per CTA
        // beyond (4096x11008, 90 panels: C = 4; 4.63 -> 4.04 us, the step
        // 0.613 -> 0.587 ms; with group-wise row scales of 128 columns,
        // whose half-panels double the panel count, C = 2: 2.88 -> 2.78 us
        // at 4096^2); C = 2 for at most 8 row blocks, else 1 (on
        // those, 64-chunk blocks make each CTA live so long that graphs of
        // such calls lose more to filling and draining than they gain; C = 2
        // on the 11 row blocks of 11008x4096 was faster alone but slower in
        // the 7B-shaped step).
        // Measured on B200 in graphs of independent calls: 28672x8192 and
        // 8192x28672 with K = 3 run 12-13% faster with 64-chunk blocks,
        // 8192^2 K = 3 9% slower, 4096^2 (the 7B-shaped matrices) slower
        // too; C = 4 on 4096^2 loses 4% in long graphs.
        long items = 0;
        for (int g : groups) items += g;
        items = items / 32 * pl.nchunks;
        if (items >= 65536 && pl.nchunks >= 2 * max_cpb) {
            set(2, 2 * max_cpb);
        } else {
            const int RB = ceil_div(pl.nchunks, max_cpb);
            set(RB <= 4 ? (pl.V <= 40 ? 1 : G == 128 ? 2 : std::min(kMaxCluster, std::max(2, (pl.V + 12) / 24)))
                        : RB <= 8 ? 2 : 1,
                ceil_div(pl.nchunks, RB));
        }
    } else {
        // Latency model of a call that waits for its predecessor (fitted to
        // dependent chains of this kernel on B200 over the shapes 4096^2,
        // 11008x4096, 4096x11008, 8192^2, 28672x8192, 8192x28672 and the
        // grouped q/k/v and gate/up calls): a CTA spends about 1 us per
        // panel on the table build, the barrier and the staging, plus 0.37
        // us per chunk of rows each warp looks up; the call takes its
        // slowest CTA's panels once per wave of clusters, a wave being what
        // fits at two CTAs per SM (90% of it: the neighbouring calls hold
        // some slots); each CTA of a cluster adds 0.2 us (the reduction, the
        // cluster's launch).  Row blocks of whole chunks per warp (8, 16, 24
        // or 32 chunks), clusters of 1, 2, 3, 4, 6, 8, 10, 12 or 16 CTAs.
        static const int kClusters[] = {1, 2, 3, 4, 6, 8, 10, 12, 16};
        int nch_max = 0;
        for (int m = 0; m < grp.n; ++m) nch_max = std::max(nch_max, round_up(grp.M[m], kChunkRows) / kChunkRows);
        double best = 1e300;
        set(1, std::min(max_cpb, pl.nchunks));
        for (int cpb = kStreamWarps; cpb <= max_cpb; cpb += kStreamWarps) {
            const int c = std::min(cpb, nch_max);
            const long RB = group_row_blocks(grp, c) * batch;
            if (RB > 65535) continue;
            const double per_chunk = 0.37 * std::ceil((double)c / kStreamWarps);
            for (int C : kClusters) {
                if (C > std::min(kMaxCluster, pl.V)) break;
                int vs[kMaxCluster + 1];
                split_weighted(groups, C, c, vs);
                double slowest = 0.0;
                for (int q = 0; q < C; ++q) {
                    double t = 0.0;
                    for (int v = vs[q]; v < vs[q + 1]; ++v) t += 1.0 + per_chunk * groups[v] / 32.0;
                    slowest = std::max(slowest, t);
                }
                const long cap = std::max(1, (int)(0.9 * cluster_capacity(sms, C)));
                const double cost = (double)ceil_div(RB, cap) * slowest + 0.2 * C;
                if (cost < best * 0.999) {
                    best = cost;
                    set(C, c);
                }
            }
            if (c == nch_max) break;
        }
    }
    if (const char *ov = getenv("FB_PLAN")) {
        int oc = 0, ocpb = 0, onw = 0;
        if (sscanf(ov, "%d,%d,%d", &oc, &ocpb, &onw) >= 2 && oc >= 1 && ocpb >= 1) {
            if (onw == 16) pl.nwarps = 16;
            set(std::min(oc, kMaxCluster), std::min(ocpb, pl.nwarps == 16 ? 4 * 16 : 8 * kStreamWarps));
        }
    }
    pl.items = stream_items(pl.cpb, pl.nwarps);
    pl.smem = stream_smem(pl.cpb);
    return pl;
}

// Plan of the batched kernel (8 warps): row blocks of up to 32 chunks, an
// even number of tokens per pass (2 for matrices of at most 32 MiB of packed
// planes, three CTAs per SM; else up to 8, two CTAs per SM; up to 16 with
// FB_PLAN's third field), and as many CTAs per cluster (up to 16) as fill
// the SMs' CTA slots once.
size_t batched_smem(int cpb, int tp) {
    return (size_t)kTableBytes + kZBytes + (size_t)tp * cpb * kChunkRows * 4;
}

Plan make_batched_plan(const fb_weights *W, int batch, int sms) {
    Plan pl;
    pl.M_pad = round_up(W->M, kChunkRows);
    pl.Pg = num_panels(W->N);
    pl.nS_pad = W->nS > 0 ? round_up(W->nS, 32) : 0;
    pl.Ps = W->nS > 0 ? num_panels(pl.nS_pad) : 0;
    const std::vector<int> groups = vpanel_groups(W->N, W->K, 0, pl.nS_pad, W->nS > 0 ? W->Ks : 0);
    pl.V = (int)groups.size();
    pl.nchunks = pl.M_pad / kChunkRows;
    pl.nwarps = kBatchWarps;
    pl.kind = 2;
    int tp_max = 8, oc = 0, ocpb = 0, otp = 0;
    const char *ov = getenv("FB_PLAN");
    const bool tuned = ov && sscanf(ov, "%d,%d,%d", &oc, &ocpb, &otp) >= 2;
    if (tuned && otp >= 2) tp_max = std::min(otp, kMaxTokensPerPass);
    // Matrices of at most 32 MiB of packed planes stay in L2 while the passes
    // stream them together, so they take passes of 2 tokens in the variant
    // with three CTAs per SM (24 warps; a pass's partials and tables fit in
    // 74 KB): more passes, but their weight reads hit L2 and the extra warps
    // hide the per-token barrier latency (8192^2 K=3 at batch 16 on B200:
    // 146.7 -> 111.9 us).  Larger ones keep passes of up to 8 tokens (two
    // CTAs per SM): for 28672x8192 passes of 2 were 4-6% slower.
    long plane_bytes = 0;
    for (int g : groups) plane_bytes += (long)g * 32 * pl.nchunks;
    pl.three = !tuned && plane_bytes <= (32L << 20) ? 1 : 0;
    if (pl.three) tp_max = 2;
    tp_max &= ~1;
    pl.tp = std::min(round_up(batch, 2), tp_max);
    pl.passes = ceil_div(batch, pl.tp);
    const int max_cpb = 4 * kBatchWarps;   // default: 4 items per warp (8 with the tuning override)
    pl.RB = ceil_div(pl.nchunks, max_cpb);
    pl.cpb = ceil_div(pl.nchunks, pl.RB);
    const long blocks = (long)pl.RB * pl.passes;
    const long slots = (pl.three ? 3L : 2L) * sms;   // fill the SMs' CTA slots once
    int C = blocks >= slots ? 1 : (int)(slots / blocks);
    C = std::max(1, std::min(std::min(C, kMaxCluster), pl.V));
    if (ov && oc >= 1 && ocpb >= 1) {
        C = std::min(std::min(oc, kMaxCluster), pl.V);
        pl.cpb = std::min(std::min(ocpb, 2 * max_cpb), pl.nchunks);
        pl.RB = ceil_div(pl.nchunks, pl.cpb);
    }
    // the cluster's partials for every token of the pass are received in the
    // table bytes: C * tp * ceil(R / C) <= tp * (R + C) floats must fit
    while (pl.cpb > 1 && (size_t)pl.tp * (pl.cpb * kChunkRows + kMaxCluster) * 4 > (size_t)kTableBytes) {
        --pl.cpb;
        pl.RB = ceil_div(pl.nchunks, pl.cpb);
    }
    pl.C = C;
    split_weighted(groups, pl.C, pl.cpb, pl.vsplit);
    pl.items = stream_items(pl.cpb);
    pl.smem = batched_smem(pl.cpb, pl.tp);
    return pl;
}

// The launch plan of a call: the batched kernel for more than one token,
// else the streaming kernel (make_stream_plan: the least work for calls
// flagged independent, the latency model for the others).
Plan make_plan(const fb_weights *W, int batch, int sms, bool independent, int G, const Group &grp) {
    if (batch > 1) return make_batched_plan(W, batch, sms);
    Plan pl = make_stream_plan(W, batch, sms, independent, G, grp);
    pl.tp = 1;
    pl.passes = 1;
    return pl;
}

const Plan &cached_plan(const fb_weights *W, int batch, int sms, bool independent, int G = 0,
                        const Group *group = nullptr) {
    struct Entry {
        PlanKey key;
        Plan plan;
    };
    thread_local Entry memo[16];
    thread_local int used = 0, next = 0;
    Group grp;
    if (group) grp = *group;
    else grp.M[0] = W->M;
    PlanKey key{W->M, W->N, W->K, W->g, W->nS, W->nS > 0 ? W->Ks : 0, batch, sms, G, independent, {0, 0, 0, 0}};
    std::copy(grp.M, grp.M + kMaxGroup, key.rows);
    for (int i = 0; i < used; ++i)
        if (memo[i].key == key) return memo[i].plan;
    Entry &e = memo[next];
    e.key = key;
    e.plan = make_plan(W, batch, sms, independent, G, grp);
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
    // all of the unified L1 / shared-memory array as shared memory, so that
    // three CTAs of ~72 KB fit on an SM (the kernels' own global loads bypass
    // or barely use L1)
    if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
        cudaSuccess)
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
    // the plan of the largest matrix (the format, hence the panels, is
    // shared), its row blocks counted over the whole group
    fb_weights Wp = *W;
    Wp.M = M_max;
    Group grp;
    grp.n = n;
    for (int m = 0; m < n; ++m) grp.M[m] = Ws[m]->M;
    const Plan &pl = cached_plan(&Wp, batch, sm_count(), (flags & FB_GEMV_INDEPENDENT) != 0, G, &grp);
    if (pl.smem > kMaxDynSmem) return FB_ERR_UNSUPPORTED;   // (no plan asks for more; a guard)
    const KernelFn fn = pl.kind == 1 ? pick_stream(t, pl.nwarps, pl.items, (flags & FB_GEMV_INDEPENDENT) != 0)
                                     : pick_batched(t, pl.items, pl.three != 0);
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
    // a cluster's CTAs on different SMs where possible: CTAs of one cluster
    // sharing an SM slow each other, and the cluster waits for its slowest
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
    const Plan &pl = cached_plan(W, batch, sms, (flags & FB_GEMV_INDEPENDENT) != 0);
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
