// lut.cu -- the two preparation steps of the FluxBin page's kernel
// (2. Kernel innovation) exposed on their own: LUT-BSF table construction
// into global memory, and the virtual columnar mapping gather.  The GEMV
// performs both inside its own kernel; these entry points let each step be
// run and checked separately.  Also: status strings and the cached SM count.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <stdint.h>

#include "fb_internal.cuh"

namespace fb {

int sm_count() {
    static std::atomic<int> cached[64];   // 0: not read yet (callers may be several host threads)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

namespace {

template <int XT>
__device__ inline float load_x(const void *x, size_t i) {
    if (XT == FB_F32) return ((const float *)x)[i];
    if (XT == FB_F16) return __half2float(((const __half *)x)[i]);
    return __bfloat162float(((const __nv_bfloat16 *)x)[i]);
}

// One thread per table entry (k, q, p):
//   lut = sum_{t<g} (bit t of p ? +1 : -1) * fp32(alpha_c * x), t ascending.
template <int XT>
__global__ void lut_build_kernel(const void *__restrict__ x, const float *__restrict__ alpha_c, int K,
                                 int N, int g, float *__restrict__ lut, size_t n_entries) {
    const int P = 1 << g, Q = N / g;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n_entries;
         e += (size_t)gridDim.x * blockDim.x) {
        const int p = (int)(e % P);
        const size_t kq = e / P;
        const int q = (int)(kq % Q), k = (int)(kq / Q);
        float s = 0.0f;
        for (int t = 0; t < g; ++t) {
            const int col = q * g + t;
            const float ac = alpha_c ? alpha_c[(size_t)k * N + col] : 1.0f;
            const float z = __fmul_rn(ac, load_x<XT>(x, col));
            s = __fadd_rn(s, ((p >> t) & 1) ? z : -z);
        }
        lut[e] = s;
    }
}

// One thread per destination element (v, t).
template <typename T>
__global__ void vcm_gather_kernel(const T *__restrict__ src, int nvec, int n_src, int ld_src,
                                  const uint32_t *__restrict__ s_idx, int nS, int nS_pad,
                                  T *__restrict__ dst, int ld_dst) {
    const size_t n = (size_t)nvec * nS_pad;
    for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
         e += (size_t)gridDim.x * blockDim.x) {
        const int v = (int)(e / nS_pad), t = (int)(e % nS_pad);
        T val;
        memset(&val, 0, sizeof val);
        if (t < nS) {
            const uint32_t j = s_idx[t];
            if (j < (uint32_t)n_src) val = src[(size_t)v * ld_src + j];
        }
        dst[(size_t)v * ld_dst + t] = val;
    }
}

int grid_for(size_t n) {
    const size_t blocks = (n + 255) / 256;
    const size_t cap = (size_t)sm_count() * 32;
    return (int)(blocks < cap ? (blocks ? blocks : 1) : cap);
}

}  // namespace
}  // namespace fb

using namespace fb;

extern "C" fb_status fb_lut_build(const void *x, fb_dtype t, const float *alpha_c, int K, int N, int g,
                                  float *lut, void *stream) {
    if (!x || !lut || !valid_dims(K, 1, N) || !(g == 1 || g == 2 || g == 4 || g == 8) || !dtype_size(t))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(x, dtype_size(t)) || !aligned(lut, 4) || (alpha_c && !aligned(alpha_c, 4)))
        return FB_ERR_MISALIGNED;
    const size_t n = (size_t)K * (N / g) * ((size_t)1 << g);
    const dim3 grid(grid_for(n)), block(256);
    cudaStream_t s = as_stream(stream);
    cudaError_t e;
    if (t == FB_F32)
        e = launch(lut_build_kernel<FB_F32>, grid, block, 0, s, false, x, alpha_c, K, N, g, lut, n);
    else if (t == FB_F16)
        e = launch(lut_build_kernel<FB_F16>, grid, block, 0, s, false, x, alpha_c, K, N, g, lut, n);
    else
        e = launch(lut_build_kernel<FB_BF16>, grid, block, 0, s, false, x, alpha_c, K, N, g, lut, n);
    return status_of(e);
}

extern "C" fb_status fb_vcm_gather(const void *src, fb_dtype t, int nvec, int n_src, int ld_src,
                                   const uint32_t *s_idx, int nS, int nS_pad, void *dst, int ld_dst,
                                   void *stream) {
    const int es = dtype_size(t);
    if (!es || nvec < 1 || n_src < 1 || ld_src < n_src || nS < 0 || nS_pad < nS || ld_dst < nS_pad ||
        !src || !dst || (nS > 0 && !s_idx))
        return FB_ERR_INVALID_VALUE;
    if (!aligned(src, es) || !aligned(dst, es) || (s_idx && !aligned(s_idx, 4))) return FB_ERR_MISALIGNED;
    const size_t n = (size_t)nvec * nS_pad;
    if (n == 0) return FB_OK;
    const dim3 grid(grid_for(n)), block(256);
    cudaStream_t s = as_stream(stream);
    cudaError_t e;
    if (es == 4)
        e = launch(vcm_gather_kernel<uint32_t>, grid, block, 0, s, false, (const uint32_t *)src, nvec,
                   n_src, ld_src, s_idx, nS, nS_pad, (uint32_t *)dst, ld_dst);
    else
        e = launch(vcm_gather_kernel<uint16_t>, grid, block, 0, s, false, (const uint16_t *)src, nvec,
                   n_src, ld_src, s_idx, nS, nS_pad, (uint16_t *)dst, ld_dst);
    return status_of(e);
}

extern "C" const char *fb_status_string(fb_status s) {
    switch (s) {
        case FB_OK: return "FB_OK";
        case FB_ERR_INVALID_VALUE: return "FB_ERR_INVALID_VALUE";
        case FB_ERR_UNSUPPORTED: return "FB_ERR_UNSUPPORTED";
        case FB_ERR_MISALIGNED: return "FB_ERR_MISALIGNED";
        case FB_ERR_WORKSPACE: return "FB_ERR_WORKSPACE";
        case FB_ERR_CUDA: return "FB_ERR_CUDA";
    }
    return "FB_ERR_UNKNOWN";
}

extern "C" int fb_abi_version(void) { return FLUXBIN_ABI_VERSION; }
