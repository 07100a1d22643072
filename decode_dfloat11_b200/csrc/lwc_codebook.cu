// Codebook decoder for sm_100a.
//
// What it computes ("Codebook Lossless Compression: когда 25% памяти значат
// больше, чем кажется", section "Как работает эта магия?"; "無損 LLM 壓縮減少
// 10-25% RAM", key points): out[i] = table[index i], where the indices are
// k-bit fields packed least significant bit first and the table holds the
// tensor's distinct 16-bit patterns.
//
// How: the table is bulk-copied (TMA engine) into a shared-memory array of
// 2^k entries, so that any k-bit field indexes inside it (entries past U are
// only reached by corrupt data and give unspecified values). The packed stream
// is cut into tiles of 1024 indices, one per warp: 32 consecutive indices per
// lane are exactly k whole 32-bit words, so every field sits at a
// compile-time bit offset. Persistent CTAs walk contiguous runs of tiles,
// possibly across several tensors of one layer; each warp keeps its own
// double buffer, filled by bulk copies two tiles ahead, and unpacks, gathers
// from the shared table and writes 16-byte stores.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "lwc_device.cuh"
#include "lwc_internal.h"

namespace lwc {
namespace {

// Warps per CTA by index width: the 32 and 64 KB tables of k = 14 and 15
// leave room for only two CTAs per SM, so those CTAs carry more warps sharing
// one copy (measured: 76-78 % of the HBM roofline instead of ~70 %). With
// k = 16 (128 KB, one CTA per SM) more warps only add contention on the
// table gathers, so it keeps 8.
template <int K>
constexpr int warps_for() { return K == 15 ? 12 : K == 14 ? 16 : 8; }
constexpr int kPerLane = 32;                            // indices per lane per tile
constexpr uint32_t kTile = 32 * kPerLane;               // indices per tile (one warp)
constexpr int kMaxBatch = 32;

struct CbTensor {
    const uint8_t *packed;
    uint64_t packed_bytes;
    const uint16_t *table;
    uint16_t *out;
    uint64_t n;
    uint64_t first_tile;   // index of this tensor's tile 0 in the launch's tile list
    uint32_t table_bytes;  // 2U rounded up to 16
    uint32_t pad;
};

struct CbBatch {
    CbTensor t[kMaxBatch];
    uint32_t count;
    uint32_t pad;
    uint64_t total_tiles;
    uint32_t *status;
};

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

template <int K>
struct CbLayout {
    static constexpr uint32_t kTileBytes = 128u * K;                       // packed bytes of one tile
    static constexpr uint32_t kTabBytes = (2u << K) < 16u ? 16u : (2u << K);
    static constexpr uint32_t kBars = 0;                                    // 2 per warp + 1 for the table
    static constexpr uint32_t kWarps = warps_for<K>();
    static constexpr uint32_t kBufs = 8 * (2 * kWarps + 2);
    static constexpr uint32_t kTab = kBufs + 2 * kWarps * kTileBytes;
    static constexpr uint32_t kTotal = kTab + kTabBytes;
};

// Lane 0: bulk copy of tile `tile` of tensor `tn` into `dst`, completing on `bar`.
template <int K>
__device__ __forceinline__ void issue_tile(const CbTensor &tn, uint64_t tile, uint32_t *dst, uint64_t *bar) {
    const uint64_t off = tile * CbLayout<K>::kTileBytes;
    const uint64_t left = tn.packed_bytes - off;
    const uint32_t bytes = (uint32_t)(left < CbLayout<K>::kTileBytes ? left : CbLayout<K>::kTileBytes);
    dev::mbar_arrive_expect_tx(bar, bytes);
    dev::bulk_g2s(dst, tn.packed + off, bytes, bar);
}

// Persistent decoder: each CTA takes a contiguous run of tiles (1024 indices
// each) from the launch's tile list; within one tensor, warp w handles tiles
// w, w + W, ... (W warps per CTA) of the run with its own double buffer and
// mbarriers, so the only CTA-wide barriers are at tensor boundaries (table
// reload).
template <int K>
__global__ void __launch_bounds__(warps_for<K>() * 32, K == 16 ? 1 : K >= 14 ? 2 : 4)   // CTAs per SM
    cb_decode_kernel(const __grid_constant__ CbBatch B) {
    using Lay = CbLayout<K>;
    constexpr uint32_t kWarps = Lay::kWarps;
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kBars);
    uint32_t *bufs = reinterpret_cast<uint32_t *>(smem + Lay::kBufs);
    uint16_t *tab = reinterpret_cast<uint16_t *>(smem + Lay::kTab);
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;

    const uint64_t t_begin = B.total_tiles * blockIdx.x / gridDim.x;
    const uint64_t t_end = B.total_tiles * (blockIdx.x + 1) / gridDim.x;
    if (t_begin >= t_end) return;

    uint64_t *tab_bar = &bars[2 * kWarps];
    uint64_t *my_bar = &bars[2 * warp];
    uint32_t *my_buf = bufs + 2 * warp * (Lay::kTileBytes / 4);
    if (tid == 0) {
        for (uint32_t i = 0; i < 2 * kWarps + 1; i++) dev::mbar_init(&bars[i], 1);
        dev::fence_mbar_init();
    }
    __syncthreads();

    uint32_t it = 0, tab_uses = 0, status = 0;
    bool dead = false;
    uint32_t ti = 0;
    uint64_t t = t_begin;
    while (t < t_end) {
        while (ti + 1 < B.count && t >= B.t[ti + 1].first_tile) ++ti;
        const CbTensor &tn = B.t[ti];
        const uint64_t seg_end = ti + 1 < B.count ? min(t_end, B.t[ti + 1].first_tile) : t_end;
        const uint64_t s0 = t - tn.first_tile, ns = seg_end - t;   // this tensor's tiles [s0, s0 + ns)

        // the tensor's table: one bulk copy, waited on by every thread
        __syncthreads();
        if (tid == 0) {
            dev::fence_proxy_async_smem();
            dev::mbar_arrive_expect_tx(tab_bar, tn.table_bytes);
            dev::bulk_g2s(tab, tn.table, tn.table_bytes, tab_bar);
        }
        // this warp's first two tiles of the run
        if (lane == 0 && !dead) {
            if (warp < ns) issue_tile<K>(tn, s0 + warp, my_buf + (it & 1u) * (Lay::kTileBytes / 4), &my_bar[it & 1u]);
            if (warp + kWarps < ns)
                issue_tile<K>(tn, s0 + warp + kWarps, my_buf + ((it + 1) & 1u) * (Lay::kTileBytes / 4),
                              &my_bar[(it + 1) & 1u]);
        }
        const bool tab_ok = dev::mbar_wait_bounded(tab_bar, tab_uses & 1u);
        tab_uses++;
        if (__syncthreads_or(!tab_ok)) {
            status |= LWC_DEVICE_TIMEOUT;
            break;
        }

        for (uint64_t j = warp; j < ns && !dead; j += kWarps, ++it) {
            const uint32_t bi = it & 1u;
            const bool ok = dev::mbar_wait_bounded(&my_bar[bi], (it >> 1) & 1u);
            if (__any_sync(0xFFFFFFFFu, !ok)) {
                // let the copy issued into the other buffer land (bounded), then stop
                status |= LWC_DEVICE_TIMEOUT;
                if (j + kWarps < ns) dev::mbar_wait_bounded(&my_bar[bi ^ 1u], ((it + 1) >> 1) & 1u);
                dead = true;
                break;
            }
            uint32_t w[K + 1];
            load_words<K>(my_buf + bi * (Lay::kTileBytes / 4) + lane * K, w);
            uint32_t o[16];
            Gather<K, 0>::run(w, tab, o);
            __syncwarp();
            if (lane == 0 && j + 2 * kWarps < ns) {
                dev::fence_proxy_async_smem();
                issue_tile<K>(tn, s0 + j + 2 * kWarps, my_buf + bi * (Lay::kTileBytes / 4), &my_bar[bi]);
            }
            const uint64_t i0 = (s0 + j) * kTile + (uint64_t)lane * kPerLane;
            if (i0 + kPerLane <= tn.n) {
                uint16_t *dst = tn.out + i0;
#pragma unroll
                for (int q = 0; q < 4; q++)
                    dev::st_v4(dst + 8 * q, make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]));
            } else {
                for (uint32_t x = 0; x < kPerLane && i0 + x < tn.n; x++)
                    tn.out[i0 + x] = (uint16_t)(o[x >> 1] >> (16 * (x & 1)));
            }
        }
        t = seg_end;
    }
    if (status && lane == 0 && B.status) atomicOr(B.status, status);
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

using KernelFn = void (*)(CbBatch);

template <int K>
constexpr KernelFn kernel_for() { return cb_decode_kernel<K>; }

const KernelFn kKernels[17] = {nullptr,          kernel_for<1>(),  kernel_for<2>(),  kernel_for<3>(),
                               kernel_for<4>(),  kernel_for<5>(),  kernel_for<6>(),  kernel_for<7>(),
                               kernel_for<8>(),  kernel_for<9>(),  kernel_for<10>(), kernel_for<11>(),
                               kernel_for<12>(), kernel_for<13>(), kernel_for<14>(), kernel_for<15>(),
                               kernel_for<16>()};

template <int K>
constexpr uint32_t smem_for() { return CbLayout<K>::kTotal; }
const int kWarpsFor[17] = {0,  warps_for<1>(),  warps_for<2>(),  warps_for<3>(),  warps_for<4>(),  warps_for<5>(),
                           warps_for<6>(),  warps_for<7>(),  warps_for<8>(),  warps_for<9>(),  warps_for<10>(),
                           warps_for<11>(), warps_for<12>(), warps_for<13>(), warps_for<14>(), warps_for<15>(),
                           warps_for<16>()};
const uint32_t kSmem[17] = {0,           smem_for<1>(),  smem_for<2>(),  smem_for<3>(),  smem_for<4>(),
                            smem_for<5>(),  smem_for<6>(),  smem_for<7>(),  smem_for<8>(),  smem_for<9>(),
                            smem_for<10>(), smem_for<11>(), smem_for<12>(), smem_for<13>(), smem_for<14>(),
                            smem_for<15>(), smem_for<16>()};

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
            err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem[k]);
            if (err == cudaSuccess)
                err = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                           cudaSharedmemCarveoutMaxShared);
            if (err == cudaSuccess)
                err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&s.per_sm[k], fn, 32 * kWarpsFor[k], kSmem[k]);
        }
        if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "device setup: %s", cudaGetErrorString(err));
        s.ready = true;
    }
    out = s;
    return LWC_OK;
}

lwc_status launch_cb_group(const std::vector<int> &idx, const lwc_desc *descs, const void *const *d_ins,
                           uint16_t *const *d_outs, uint32_t *d_status, cudaStream_t stream, const DevState &ds) {
    CbBatch B;
    std::memset(&B, 0, sizeof B);
    const uint32_t K = descs[idx[0]].k;
    uint64_t tiles = 0;
    for (size_t j = 0; j < idx.size(); j++) {
        const lwc_desc &d = descs[idx[j]];
        const uint8_t *base = static_cast<const uint8_t *>(d_ins[idx[j]]);
        CbTensor &t = B.t[j];
        t.packed = base + d.off_packed;
        t.packed_bytes = d.packed_bytes;
        t.table = reinterpret_cast<const uint16_t *>(base + d.off_table);
        t.table_bytes = (uint32_t)((2ull * d.U + 15) / 16 * 16);
        t.out = d_outs[idx[j]];
        t.n = d.n;
        t.first_tile = tiles;
        tiles += (d.n + kTile - 1) / kTile;
    }
    B.count = (uint32_t)idx.size();
    B.total_tiles = tiles;
    B.status = d_status;
    const int per_sm = std::max(1, ds.per_sm[K]);
    const uint32_t warps = (uint32_t)kWarpsFor[K];
    // enough CTAs that every warp of every resident CTA gets tiles
    const uint64_t grid = std::min<uint64_t>((tiles + warps - 1) / warps, (uint64_t)per_sm * ds.sms);
    kKernels[K]<<<(unsigned)grid, 32 * warps, kSmem[K], stream>>>(B);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
    return LWC_OK;
}

}  // namespace
}  // namespace lwc

using namespace lwc;

extern "C" {

lwc_status lwc_decode_codebook_batched(const lwc_desc *descs, const void *const *d_ins, uint16_t *const *d_outs,
                                       int count, uint32_t *d_status, lwc_stream_t stream) {
    if (count < 0 || (count > 0 && (!descs || !d_ins || !d_outs)))
        return fail(LWC_ERR_INVALID_ARG, "bad batch arguments");
    bool any = false;
    for (int i = 0; i < count; i++) {
        lwc_status st = check_codebook_desc(&descs[i]);
        if (st) return st;
        if (descs[i].n == 0) continue;
        any = true;
        if (!d_ins[i] || !d_outs[i]) return fail(LWC_ERR_INVALID_ARG, "NULL device pointer (tensor %d)", i);
        if (!aligned16(d_ins[i]) || !aligned16(d_outs[i]))
            return fail(LWC_ERR_MISALIGNED, "device pointers must be 16-byte aligned (tensor %d)", i);
    }
    if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u))
        return fail(LWC_ERR_MISALIGNED, "status word must be 4-byte aligned");
    if (!any) {
        clear_error();
        return LWC_OK;
    }
    DevState ds;
    lwc_status st = device_state(ds);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one-entry tables: a fill; the rest grouped by index width
    std::vector<std::vector<int>> by_k(17);
    for (int i = 0; i < count; i++) {
        const lwc_desc &d = descs[i];
        if (d.n == 0) continue;
        if (d.k == 0) {
            const uint64_t blocks = std::min<uint64_t>((d.n + 8 * 256 - 1) / (8 * 256), (uint64_t)ds.sms * 8);
            cb_fill_kernel<<<(unsigned)blocks, 256, 0, s>>>(
                d_outs[i], d.n, reinterpret_cast<const uint16_t *>(static_cast<const uint8_t *>(d_ins[i]) + d.off_table));
            cudaError_t err = cudaGetLastError();
            if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
            continue;
        }
        by_k[d.k].push_back(i);
    }
    for (int k = 1; k <= 16; k++) {
        for (size_t a = 0; a < by_k[k].size(); a += kMaxBatch) {
            std::vector<int> g(by_k[k].begin() + a, by_k[k].begin() + std::min(by_k[k].size(), a + kMaxBatch));
            st = launch_cb_group(g, descs, d_ins, d_outs, d_status, s, ds);
            if (st) return st;
        }
    }
    clear_error();
    return LWC_OK;
}

lwc_status lwc_decode_codebook_checked(const lwc_desc *desc, const void *d_in, uint16_t *d_out, uint32_t *d_status,
                                       lwc_stream_t stream) {
    if (!desc) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    return lwc_decode_codebook_batched(desc, &d_in, &d_out, 1, d_status, stream);
}

lwc_status lwc_decode_codebook(const lwc_desc *desc, const void *d_in, uint16_t *d_out, lwc_stream_t stream) {
    return lwc_decode_codebook_checked(desc, d_in, d_out, nullptr, stream);
}

}  // extern "C"
