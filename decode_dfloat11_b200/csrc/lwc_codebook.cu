// Codebook decoder for sm_100a.
//
// What it computes ("Codebook Lossless Compression: когда 25% памяти значат
// больше, чем кажется", section "Как работает эта магия?"; "無損 LLM 壓縮減少
// 10-25% RAM", key points): out[i] = table[index i], where the indices are
// k-bit fields packed least significant bit first and the table holds the
// tensor's distinct 16-bit patterns.
//
// How: the table is copied once per CTA into shared memory, padded with zeros
// to 2^k entries so that any k-bit field is a valid index. The packed stream
// is cut into tiles of 32 * T indices (T threads, 32 consecutive indices per
// thread = k whole 32-bit words, so every field sits at a compile-time bit
// offset). Persistent CTAs walk contiguous runs of tiles; one thread issues a
// bulk copy (TMA engine) of the next tile into the other half of a double
// buffer while all threads unpack, gather from the shared table and write the
// current one with 16-byte stores.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "lwc_device.cuh"
#include "lwc_internal.h"

namespace lwc {
namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 32;                       // indices per thread per tile
constexpr uint32_t kTile = kThreads * kPerThread;    // indices per tile

struct CbArgs {
    const uint32_t *packed;   // packed words
    uint64_t packed_bytes;
    const uint16_t *table;
    uint32_t U;
    uint16_t *out;
    uint64_t n;
    uint64_t n_tiles;
    uint32_t *status;
};

// Load a thread's K words from shared memory, as wide as their alignment allows.
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
    constexpr uint32_t mask = (K == 32) ? 0xFFFFFFFFu : ((1u << K) - 1u);
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

template <int K>
__global__ void __launch_bounds__(kThreads) cb_decode_kernel(const __grid_constant__ CbArgs A) {
    extern __shared__ __align__(16) uint8_t smem[];
    constexpr uint32_t kTabEntries = 1u << K;
    constexpr uint32_t kTileWords = kThreads * K;    // 32 fields of K bits per thread = K words
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem);                 // 2 mbarriers
    uint32_t *tiles = reinterpret_cast<uint32_t *>(smem + 16);          // 2 x kTileWords
    uint16_t *tab = reinterpret_cast<uint16_t *>(smem + 16 + 8 * kTileWords);

    const uint32_t tid = threadIdx.x;
    const uint64_t t_begin = A.n_tiles * blockIdx.x / gridDim.x;
    const uint64_t t_end = A.n_tiles * (blockIdx.x + 1) / gridDim.x;
    if (t_begin >= t_end) return;

    auto issue = [&](uint64_t t, uint32_t buf) {
        const uint64_t off = t * (uint64_t)kTileWords * 4;
        const uint64_t left = A.packed_bytes - off;
        const uint32_t bytes = (uint32_t)(left < (uint64_t)kTileWords * 4 ? left : (uint64_t)kTileWords * 4);
        dev::mbar_arrive_expect_tx(&bars[buf], bytes);
        dev::bulk_g2s(tiles + buf * kTileWords, reinterpret_cast<const uint8_t *>(A.packed) + off, bytes, &bars[buf]);
    };

    if (tid == 0) {
        dev::mbar_init(&bars[0], 1);
        dev::mbar_init(&bars[1], 1);
        dev::fence_mbar_init();
        issue(t_begin, 0);
    }
    for (uint32_t i = tid; i < kTabEntries; i += kThreads) tab[i] = i < A.U ? A.table[i] : (uint16_t)0;
    __syncthreads();

    uint32_t timed_out = 0;
    for (uint64_t t = t_begin; t < t_end; ++t) {
        const uint32_t it = (uint32_t)(t - t_begin), buf = it & 1u;
        if (tid == 0 && t + 1 < t_end) {
            dev::fence_proxy_async_smem();
            issue(t + 1, buf ^ 1u);
        }
        const bool ok = dev::mbar_wait_bounded(&bars[buf], (it >> 1) & 1u);
        if (__syncthreads_or(!ok)) {
            // let the copy already issued for the next tile land (bounded) before leaving
            timed_out = 1;
            if (t + 1 < t_end) dev::mbar_wait_bounded(&bars[buf ^ 1u], ((it + 1) >> 1) & 1u);
            break;
        }
        uint32_t w[K + 1];
        load_words<K>(tiles + buf * kTileWords + tid * K, w);
        uint32_t o[16];
        Gather<K, 0>::run(w, tab, o);
        const uint64_t i0 = t * kTile + (uint64_t)tid * kPerThread;
        if (i0 + kPerThread <= A.n) {
            uint16_t *dst = A.out + i0;
#pragma unroll
            for (int q = 0; q < 4; q++) dev::st_v4(dst + 8 * q, make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]));
        } else {
            for (uint32_t j = 0; j < kPerThread && i0 + j < A.n; j++)
                A.out[i0 + j] = (uint16_t)(o[j >> 1] >> (16 * (j & 1)));
        }
        __syncthreads();   // every thread is done with `buf` before it is refilled
    }
    if (timed_out && tid == 0 && A.status) atomicOr(A.status, LWC_DEVICE_TIMEOUT);
}

// U == 1: every weight is the single table entry.
__global__ void cb_fill_kernel(uint16_t *__restrict__ out, uint64_t n, const uint16_t *__restrict__ table) {
    const uint32_t v = table[0];
    const uint32_t vv = v | (v << 16);
    const uint64_t stride = 8ull * gridDim.x * blockDim.x;
    for (uint64_t g = 8ull * (blockIdx.x * (uint64_t)blockDim.x + threadIdx.x); g < n; g += stride) {
        if (g + 8 <= n)
            dev::st_v4(out + g, make_uint4(vv, vv, vv, vv));
        else
            for (uint64_t i = g; i < n; i++) out[i] = (uint16_t)v;
    }
}

using KernelFn = void (*)(CbArgs);

template <int K>
constexpr KernelFn kernel_for() { return cb_decode_kernel<K>; }

const KernelFn kKernels[17] = {nullptr,          kernel_for<1>(),  kernel_for<2>(),  kernel_for<3>(),
                               kernel_for<4>(),  kernel_for<5>(),  kernel_for<6>(),  kernel_for<7>(),
                               kernel_for<8>(),  kernel_for<9>(),  kernel_for<10>(), kernel_for<11>(),
                               kernel_for<12>(), kernel_for<13>(), kernel_for<14>(), kernel_for<15>(),
                               kernel_for<16>()};

uint64_t smem_bytes(uint32_t k) { return 16 + 8ull * kThreads * k + 2ull * (1u << k); }

struct DevState {
    int sms = 0;
    int per_sm[17] = {0};
    bool ready = false;
};
std::mutex g_mutex;
std::vector<DevState> g_dev;

lwc_status device_state(DevState &out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
    std::lock_guard<std::mutex> lock(g_mutex);
    if ((int)g_dev.size() <= dev) g_dev.resize(dev + 1);
    DevState &s = g_dev[dev];
    if (!s.ready) {
        err = cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev);
        for (int k = 1; k <= 16 && err == cudaSuccess; k++) {
            const void *fn = (const void *)kKernels[k];
            err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(k));
            if (err == cudaSuccess)
                err = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                           cudaSharedmemCarveoutMaxShared);
            if (err == cudaSuccess)
                err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&s.per_sm[k], fn, kThreads, smem_bytes(k));
        }
        if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "device setup: %s", cudaGetErrorString(err));
        s.ready = true;
    }
    out = s;
    return LWC_OK;
}

}  // namespace
}  // namespace lwc

using namespace lwc;

extern "C" {

lwc_status lwc_decode_codebook_checked(const lwc_desc *desc, const void *d_in, uint16_t *d_out, uint32_t *d_status,
                                       lwc_stream_t stream) {
    lwc_status st = check_codebook_desc(desc);
    if (st) return st;
    if (desc->n == 0) {
        clear_error();
        return LWC_OK;
    }
    if (!d_in || !d_out) return fail(LWC_ERR_INVALID_ARG, "NULL device pointer");
    if (!aligned16(d_in) || !aligned16(d_out)) return fail(LWC_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
    if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u))
        return fail(LWC_ERR_MISALIGNED, "status word must be 4-byte aligned");
    DevState ds;
    st = device_state(ds);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint8_t *base = static_cast<const uint8_t *>(d_in);
    const uint16_t *table = reinterpret_cast<const uint16_t *>(base + desc->off_table);
    if (desc->k == 0) {
        const uint64_t blocks = std::min<uint64_t>((desc->n + 8 * 256 - 1) / (8 * 256), (uint64_t)ds.sms * 8);
        cb_fill_kernel<<<(unsigned)blocks, 256, 0, s>>>(d_out, desc->n, table);
    } else {
        CbArgs A;
        A.packed = reinterpret_cast<const uint32_t *>(base + desc->off_packed);
        A.packed_bytes = desc->packed_bytes;
        A.table = table;
        A.U = desc->U;
        A.out = d_out;
        A.n = desc->n;
        A.n_tiles = (desc->n + kTile - 1) / kTile;
        A.status = d_status;
        const int per_sm = std::max(1, ds.per_sm[desc->k]);
        const uint64_t grid = std::min<uint64_t>(A.n_tiles, (uint64_t)per_sm * ds.sms);
        kKernels[desc->k]<<<(unsigned)grid, kThreads, (size_t)smem_bytes(desc->k), s>>>(A);
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
    clear_error();
    return LWC_OK;
}

lwc_status lwc_decode_codebook(const lwc_desc *desc, const void *d_in, uint16_t *d_out, lwc_stream_t stream) {
    return lwc_decode_codebook_checked(desc, d_in, d_out, nullptr, stream);
}

}  // extern "C"
