// fb_internal.cuh -- internal helpers shared by the library's .cu files:
// the device weight layout of include/fluxbin.h, argument checks, launch
// plumbing.  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fluxbin.h"

namespace fb {

constexpr int kPanelCols = 256;   // columns per panel
constexpr int kChunkRows = 32;    // rows per chunk (one row per lane)
constexpr int kMaxM = 1 << 24;
constexpr int kMaxN = 1 << 20;
constexpr int kMaxK = 4;
constexpr int kMaxBatch = 64;

__host__ __device__ inline int round_up(int a, int b) { return (a + b - 1) / b * b; }
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Number of panels of an N-column matrix, and the width of panel p.
__host__ __device__ inline int num_panels(int N) { return ceil_div(N, kPanelCols); }
__host__ __device__ inline int panel_width(int N, int p) {
    int w = N - p * kPanelCols;
    return w < kPanelCols ? w : kPanelCols;
}

// Byte offset, inside a chunk block, of stored position u of lane l.
__host__ __device__ inline int position_offset(int u, int l, int Bp) {
    return (Bp % 16 == 0) ? (u / 16) * 512 + 16 * l + (u % 16) : (u / 4) * 128 + 4 * l + (u % 4);
}

// Inverse of position_offset for a 4-byte aligned offset o: the lane and the
// first of the four positions held by that 32-bit word.
__host__ __device__ inline void word_position(int o, int Bp, int *lane, int *u0) {
    if (Bp % 16 == 0) {
        const int seg = o / 512, rem = o % 512;
        *lane = rem / 16;
        *u0 = seg * 16 + (rem % 16);
    } else {
        const int seg = o / 128, rem = o % 128;
        *lane = rem / 4;
        *u0 = seg * 4;
    }
}

inline bool valid_dims(int K, int M, int N) {
    return K >= 1 && K <= kMaxK && M >= 1 && M <= kMaxM && N >= 32 && N <= kMaxN && N % 32 == 0;
}

inline bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

inline int dtype_size(fb_dtype t) { return t == FB_F32 ? 4 : (t == FB_F16 || t == FB_BF16) ? 2 : 0; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// SM count of the current device (cached per device).
int sm_count();

// Launch through cudaLaunchKernelEx so the launch's own status comes back
// (no reliance on the thread's last-error slot).  pdl = programmatic
// dependent launch (the kernel may start before the previous one ends).
template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, bool pdl, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

inline fb_status status_of(cudaError_t e) { return e == cudaSuccess ? FB_OK : FB_ERR_CUDA; }

}  // namespace fb
