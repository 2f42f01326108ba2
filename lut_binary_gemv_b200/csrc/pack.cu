// pack.cu -- load-time packing of +/-1 sign planes into the device layout of
// include/fluxbin.h (the "compressed Uint32 weights" that the FluxBin page's
// kernel streams, 2. Kernel innovation, execution flow), and the inverse.
#include <cuda_runtime.h>
#include <stdint.h>

#include "fb_internal.cuh"

namespace fb {
namespace {

enum class Src { kInt8Signs, kCanonicalBits };

// Where one 32-bit word of the planes buffer comes from.
struct WordSite {
    int k, p, c, lane, u0, Bp;
};

__device__ inline WordSite decode_word(size_t wi, int M_pad, int N) {
    const size_t base_bytes = (size_t)M_pad * (N / 8);
    size_t o = wi * 4;
    WordSite s;
    s.k = (int)(o / base_bytes);
    o -= (size_t)s.k * base_bytes;
    s.p = (int)(o / ((size_t)32 * M_pad));
    o -= (size_t)32 * s.p * M_pad;
    s.Bp = panel_width(N, s.p) / 8;
    s.c = (int)(o / ((size_t)32 * s.Bp));
    const int o3 = (int)(o - (size_t)32 * s.Bp * s.c);
    word_position(o3, s.Bp, &s.lane, &s.u0);
    return s;
}

template <Src S>
__global__ void pack_kernel(const void *__restrict__ src, int K, int M, int N, int M_pad,
                            uint32_t *__restrict__ planes, size_t nwords) {
    for (size_t wi = blockIdx.x * (size_t)blockDim.x + threadIdx.x; wi < nwords;
         wi += (size_t)gridDim.x * blockDim.x) {
        const WordSite s = decode_word(wi, M_pad, N);
        const int row = s.c * kChunkRows + s.lane;
        uint32_t word = 0;
        if (row < M) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int q = (s.lane + s.u0 + j) % s.Bp;      // byte group held at position u0+j
                const int col = s.p * kPanelCols + 8 * q;
                uint32_t byte = 0;
                if (S == Src::kInt8Signs) {
                    const int8_t *r = (const int8_t *)src + ((size_t)s.k * M + row) * (size_t)N + col;
                    const uint2 v = *reinterpret_cast<const uint2 *>(r);   // 8 signs, 8-byte aligned
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        const int8_t sg = (int8_t)(((t < 4 ? v.x : v.y) >> (8 * (t & 3))) & 0xFF);
                        byte |= (uint32_t)(sg > 0) << t;
                    }
                } else {
                    byte = ((const uint8_t *)src)[((size_t)s.k * M + row) * (size_t)(N / 8) + col / 8];
                }
                word |= byte << (8 * j);
            }
        }
        planes[wi] = word;
    }
}

__global__ void unpack_kernel(const uint32_t *__restrict__ planes, int K, int M, int N, int M_pad,
                              int8_t *__restrict__ signs, size_t nwords) {
    for (size_t wi = blockIdx.x * (size_t)blockDim.x + threadIdx.x; wi < nwords;
         wi += (size_t)gridDim.x * blockDim.x) {
        const WordSite s = decode_word(wi, M_pad, N);
        const int row = s.c * kChunkRows + s.lane;
        if (row >= M) continue;
        const uint32_t word = planes[wi];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int q = (s.lane + s.u0 + j) % s.Bp;
            const int col = s.p * kPanelCols + 8 * q;
            int8_t *r = signs + ((size_t)s.k * M + row) * (size_t)N + col;
#pragma unroll
            for (int t = 0; t < 8; ++t) r[t] = ((word >> (8 * j + t)) & 1) ? 1 : -1;
        }
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

extern "C" size_t fb_packed_words(int K, int M, int N) {
    if (!valid_dims(K, M, N)) return 0;
    return (size_t)K * round_up(M, kChunkRows) * (size_t)N / 32;
}

template <Src S>
static fb_status pack_common(const void *src, int K, int M, int N, uint32_t *planes, void *stream) {
    if (!src || !planes || !valid_dims(K, M, N)) return FB_ERR_INVALID_VALUE;
    if (!aligned(planes, 16) || (S == Src::kInt8Signs && !aligned(src, 8)))
        return FB_ERR_MISALIGNED;
    const size_t n = fb_packed_words(K, M, N);
    return status_of(launch(pack_kernel<S>, dim3(grid_for(n)), dim3(256), 0, as_stream(stream), false,
                            src, K, M, N, round_up(M, kChunkRows), planes, n));
}

extern "C" fb_status fb_pack(const int8_t *signs, int K, int M, int N, uint32_t *planes, void *stream) {
    return pack_common<Src::kInt8Signs>(signs, K, M, N, planes, stream);
}

extern "C" fb_status fb_pack_bits(const uint8_t *bits, int K, int M, int N, uint32_t *planes,
                                  void *stream) {
    return pack_common<Src::kCanonicalBits>(bits, K, M, N, planes, stream);
}

extern "C" fb_status fb_unpack(const uint32_t *planes, int K, int M, int N, int8_t *signs, void *stream) {
    if (!planes || !signs || !valid_dims(K, M, N)) return FB_ERR_INVALID_VALUE;
    if (!aligned(planes, 16)) return FB_ERR_MISALIGNED;
    const size_t n = fb_packed_words(K, M, N);
    return status_of(launch(unpack_kernel, dim3(grid_for(n)), dim3(256), 0, as_stream(stream), false,
                            planes, K, M, N, round_up(M, kChunkRows), signs, n));
}
