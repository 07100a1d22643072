// Device code shared by the codebook kernels (the decoder and fused linear
// layer of lwc_codebook.cu, the tensor-core product of lwc_gemm.cu): a lane
// holds 32 consecutive k-bit indices, which are exactly k whole 32-bit words
// (packed least significant bit first), so every field sits at a
// compile-time bit offset; the 32 values are gathered from the shared-memory
// table in pairs.
//
// What it computes ("Codebook Lossless Compression: когда 25% памяти значат
// больше, чем кажется", section "Как работает эта магия?"): out[i] =
// table[index i].
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace lwc {
namespace cbdev {

// Load a lane's K words from shared memory, as wide as their alignment allows.
template <int K>
__device__ __forceinline__ void load_words(const uint32_t *src, uint32_t (&w)[K + 1]) {
    if constexpr (K % 4 == 0) {
#pragma unroll
        for (int i = 0; i < K / 4; i++) {
            const uint4 v = reinterpret_cast<const uint4 *>(src)[i];
            w[4 * i] = v.x;
            w[4 * i + 1] = v.y;
            w[4 * i + 2] = v.z;
            w[4 * i + 3] = v.w;
        }
    } else if constexpr (K % 2 == 0) {
#pragma unroll
        for (int i = 0; i < K / 2; i++) {
            const uint2 v = reinterpret_cast<const uint2 *>(src)[i];
            w[2 * i] = v.x;
            w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < K; i++) w[i] = src[i];
    }
    w[K] = 0;
}

// Field j of width K starting at bit j*K of the word array (compile-time offsets).
template <int K, int J>
__device__ __forceinline__ uint32_t field(const uint32_t (&w)[K + 1]) {
    constexpr int bit = J * K, word = bit >> 5, sh = bit & 31;
    constexpr uint32_t mask = (1u << K) - 1u;
    if constexpr (sh + K <= 32)
        return (w[word] >> sh) & mask;
    else
        return __funnelshift_r(w[word], w[word + 1], sh) & mask;
}

template <int K, int J>
struct Gather {
    __device__ __forceinline__ static void run(const uint32_t (&w)[K + 1], const uint16_t *tab, uint32_t (&o)[16]) {
        const uint32_t a = tab[field<K, J>(w)];
        const uint32_t b = tab[field<K, J + 1>(w)];
        o[J / 2] = a | (b << 16);
        Gather<K, J + 2>::run(w, tab, o);
    }
};
template <int K>
struct Gather<K, 32> {
    __device__ __forceinline__ static void run(const uint32_t (&)[K + 1], const uint16_t *, uint32_t (&)[16]) {}
};

}  // namespace cbdev
}  // namespace lwc
