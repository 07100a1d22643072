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
//
// Also here: cb_linear_kernel, the decode fused into the linear layer that
// consumes the weights (y = x W^T for up to 8 activation rows, weights kept
// in registers; see the section comment below), and the self-test kernel of
// the bounded mbarrier wait all these kernels use.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "lwc_cb_dev.cuh"
#include "lwc_device.cuh"
#include "lwc_internal.h"

namespace lwc {
namespace {

using namespace cbdev;

// Warps per CTA by index width: the 32 and 64 KB tables of k = 14 and 15
// leave room for only two CTAs per SM, so those CTAs carry more warps sharing
// one copy (measured: 76-78 % of the HBM roofline instead of ~70 %). With
// k = 16 (128 KB, one CTA per SM) more warps only add contention on the
// table gathers, so it keeps 8.
template <int K>
constexpr int warps_for() { return K == 15 ? 12 : K == 14 ? 16 : 8; }
// Tile buffers per warp (bulk copies in flight per warp). Measured on
// 256M-weight tensors: a third buffer lifts k = 14 and 15 (whose 2-CTA SMs
// have few warps) from 76-78 % to 84-88 % of the HBM roofline; it costs k = 13
// a few points and does not help k = 16.
template <int K>
constexpr int bufs_for() { return K == 14 || K == 15 ? 3 : 2; }
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

template <int K>
struct CbLayout {
    static constexpr uint32_t kTileBytes = 128u * K;                       // packed bytes of one tile
    static constexpr uint32_t kTabBytes = (2u << K) < 16u ? 16u : (2u << K);
    static constexpr uint32_t kBars = 0;                                    // NB per warp + 1 for the table
    static constexpr uint32_t kWarps = warps_for<K>();
    static constexpr uint32_t NB = bufs_for<K>();
    static constexpr uint32_t kBufs = (8 * (NB * kWarps + 1) + 15) / 16 * 16;
    static constexpr uint32_t kTab = kBufs + NB * kWarps * kTileBytes;
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
// w, w + W, ... (W warps per CTA) of the run with its own NB tile buffers
// (copies issued NB tiles ahead) and mbarriers, so the only CTA-wide barriers
// are at tensor boundaries (table reload).
template <int K>
__global__ void __launch_bounds__(warps_for<K>() * 32, K == 16 ? 1 : K >= 14 ? 2 : 4)   // CTAs per SM
    cb_decode_kernel(const __grid_constant__ CbBatch B) {
    using Lay = CbLayout<K>;
    constexpr uint32_t kWarps = Lay::kWarps, NB = Lay::NB;
    constexpr uint32_t kTileWords = Lay::kTileBytes / 4;
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kBars);
    uint32_t *bufs = reinterpret_cast<uint32_t *>(smem + Lay::kBufs);
    uint16_t *tab = reinterpret_cast<uint16_t *>(smem + Lay::kTab);
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;

    const uint64_t t_begin = B.total_tiles * blockIdx.x / gridDim.x;
    const uint64_t t_end = B.total_tiles * (blockIdx.x + 1) / gridDim.x;
    if (t_begin >= t_end) return;

    uint64_t *tab_bar = &bars[NB * kWarps];
    uint64_t *my_bar = &bars[NB * warp];
    uint32_t *my_buf = bufs + NB * warp * kTileWords;
    if (tid == 0) {
        for (uint32_t i = 0; i < NB * kWarps + 1; i++) dev::mbar_init(&bars[i], 1);
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
        // this warp's first NB tiles of the run (use u of buffer b completes phase u & 1 of its mbarrier)
        if (lane == 0 && !dead) {
            dev::fence_proxy_async_smem();   // this warp's reads of its buffers come before the copies' writes
#pragma unroll
            for (uint32_t q = 0; q < NB; q++)
                if (warp + q * kWarps < ns)
                    issue_tile<K>(tn, s0 + warp + q * kWarps, my_buf + ((it + q) % NB) * kTileWords,
                                  &my_bar[(it + q) % NB]);
        }
        const bool tab_ok = dev::mbar_wait_bounded(tab_bar, tab_uses & 1u);
        tab_uses++;
        if (__syncthreads_or(!tab_ok)) {
            // let the table copy and this warp's first tiles land (bounded), then stop
            status |= LWC_DEVICE_TIMEOUT;
            if (tid == 0) dev::mbar_wait_bounded(tab_bar, (tab_uses - 1) & 1u);
            if (!dead)
                for (uint32_t q = 0; q < NB; q++)
                    if (warp + q * kWarps < ns) dev::mbar_wait_bounded(&my_bar[(it + q) % NB], ((it + q) / NB) & 1u);
            break;
        }

        for (uint64_t j = warp; j < ns && !dead; j += kWarps, ++it) {
            const uint32_t bi = it % NB;
            const bool ok = dev::mbar_wait_bounded(&my_bar[bi], (it / NB) & 1u);
            if (__any_sync(0xFFFFFFFFu, !ok)) {
                // let this tile's copy and the ones issued into the other buffers land (bounded), then stop
                status |= LWC_DEVICE_TIMEOUT;
                for (uint32_t q = 0; q < NB; q++)
                    if (j + q * kWarps < ns) dev::mbar_wait_bounded(&my_bar[(it + q) % NB], ((it + q) / NB) & 1u);
                dead = true;
                break;
            }
            uint32_t w[K + 1];
            load_words<K>(my_buf + bi * kTileWords + lane * K, w);
            uint32_t o[16];
            Gather<K, 0>::run(w, tab, o);
            __syncwarp();
            if (lane == 0 && j + NB * kWarps < ns) {
                dev::fence_proxy_async_smem();
                issue_tile<K>(tn, s0 + j + NB * kWarps, my_buf + bi * kTileWords, &my_bar[bi]);
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

// U == 65536: the table holds every 16-bit pattern in ascending order, so
// table[j] = j and out[i] = index i: the packed 16-bit fields (least
// significant bit first) are the weights themselves, little-endian. The
// decode is a copy, 64 bytes per thread step; the CTAs also check the table
// (a slice each) and report LWC_DEVICE_BAD_CODE if it is not the identity.
__global__ void __launch_bounds__(256) cb_identity_kernel(const uint8_t *__restrict__ packed, uint16_t *__restrict__ out,
                                                          uint64_t n, const uint16_t *__restrict__ table,
                                                          uint32_t *status) {
    const uint64_t tid = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x, nt = (uint64_t)gridDim.x * blockDim.x;
    uint32_t bad = 0;
    for (uint64_t j = tid; j < 65536; j += nt) bad |= table[j] != (uint16_t)j;
    const uint4 *src = reinterpret_cast<const uint4 *>(packed);
    uint4 *dst = reinterpret_cast<uint4 *>(out);
    const uint64_t n16 = n / 8;   // whole 16-byte groups of 8 weights
    uint64_t g = tid;
    for (; g + 3 * nt < n16; g += 4 * nt) {
        const uint4 a = __ldg(src + g), b = __ldg(src + g + nt), c = __ldg(src + g + 2 * nt), d = __ldg(src + g + 3 * nt);
        dst[g] = a;
        dst[g + nt] = b;
        dst[g + 2 * nt] = c;
        dst[g + 3 * nt] = d;
    }
    for (; g < n16; g += nt) dst[g] = __ldg(src + g);
    const uint16_t *src16 = reinterpret_cast<const uint16_t *>(packed);
    for (uint64_t i = 8 * n16 + tid; i < n; i += nt) out[i] = src16[i];
    if (bad && status) atomicOr(status, LWC_DEVICE_BAD_CODE);
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

// ---- fused decode + linear layer ---------------------------------------------
//
// y[m, r] = sum_c W[r, c] x[m, c] for M <= 8 activation rows, with W the
// tensor's rows x cols weights, decoded in registers and never written out.
// One warp owns one row at a time and walks it in windows of 1024 indices
// (32 per lane); each window's packed bits are bulk-copied from the
// 16-byte boundary at or below its first bit, and every lane re-aligns its K
// + 1 words by the window's bit offset (the same for all lanes, since 32
// fields are K whole words), so the fields keep compile-time positions for
// any cols. Each lane sums its 32 products of a window in FP32 as one FMA
// chain per activation row and adds that to its running sum for the row; a
// 5-level butterfly sums the lanes, and lane 0 stores the row's outputs: the
// summation tree has height at most ceil(cols / 1024) + 37, and the result
// does not depend on the launch shape.

constexpr int kMaxRows = 8;          // activation rows per call
constexpr uint32_t kLinWarps = 8;    // warps per CTA
constexpr uint32_t kXStageMax = 65536;   // shared-memory bytes for a tensor's activations (M x whole windows)

struct CbLinTensor {
    const uint8_t *packed;
    uint64_t packed_bytes;
    const uint16_t *table;
    const uint16_t *x;     // M x cols BF16, row-major
    float *y;              // M x rows FP32, row-major
    uint64_t rows;
    uint64_t first_row;    // index of this tensor's row 0 in the launch's row list
    uint64_t first_win;    // index of its first window in the launch's window list
    uint32_t cols;
    uint32_t table_bytes;
    uint32_t stage_x;      // 1: the CTA copies x into shared memory (fits kXStageMax)
    uint32_t pad;
};

struct CbLinBatch {
    CbLinTensor t[kMaxBatch];
    uint32_t count;
    uint32_t M;
    uint32_t x_stage_bytes;   // shared memory after the table for staged activations
    uint64_t total_rows;
    uint64_t total_wins;
    uint32_t *status;
};

// The first row (in the launch's row list) whose first window is at or after
// window u: CTAs take equal runs of windows, rounded to whole rows.
__device__ __forceinline__ uint64_t row_at_window(const CbLinBatch &B, uint64_t u) {
    if (u >= B.total_wins) return B.total_rows;
    uint32_t t = 0;
    while (t + 1 < B.count && B.t[t + 1].first_win <= u) ++t;
    const CbLinTensor &tn = B.t[t];
    const uint32_t nwin = (tn.cols + kTile - 1) / kTile;
    return tn.first_row + (u - tn.first_win + nwin - 1) / nwin;
}

template <int K>
struct CbLinLayout {
    // a window's 128 K bytes from the aligned start at or below its first bit
    // (at most 15 bytes earlier), plus the word after its last field
    static constexpr uint32_t kBufBytes = 128u * K + 48u;
    static constexpr uint32_t kTabBytes = (2u << K) < 16u ? 16u : (2u << K);
    static constexpr uint32_t kWarps = kLinWarps;
    static constexpr uint32_t kBars = 0;
    static constexpr uint32_t kBufs = 8 * (2 * kWarps + 2);
    static constexpr uint32_t kTab = kBufs + 2 * kWarps * kBufBytes;
    static constexpr uint32_t kTotal = kTab + kTabBytes;
};

// Index range of window q of row r: first index and count.
__device__ __forceinline__ uint64_t window_first(const CbLinTensor &tn, uint64_t r, uint32_t q) {
    return r * tn.cols + (uint64_t)q * kTile;
}
__device__ __forceinline__ uint32_t window_count(const CbLinTensor &tn, uint32_t q) {
    return min(kTile, tn.cols - q * kTile);
}

// Lane 0: bulk copy of window q of row r into dst, completing on bar.
template <int K>
__device__ __forceinline__ void issue_window(const CbLinTensor &tn, uint64_t r, uint32_t q, uint32_t *dst,
                                             uint64_t *bar) {
    const uint64_t bit0 = window_first(tn, r, q) * K;
    const uint64_t a0 = (bit0 >> 3) & ~15ull;
    const uint64_t need = (bit0 + (uint64_t)window_count(tn, q) * K + 7) / 8 + 4;   // through the next word
    uint64_t end = (need + 15) & ~15ull;
    if (end > tn.packed_bytes) end = tn.packed_bytes;   // the words past the section are never used
    const uint32_t bytes = (uint32_t)(end - a0);
    dev::mbar_arrive_expect_tx(bar, bytes);
    dev::bulk_g2s(dst, tn.packed + a0, bytes, bar);
}

__device__ __forceinline__ float bf16_lo(uint32_t p) { return __uint_as_float(p << 16); }

// acc + w.lo * x.lo, then + w.hi * x.hi: two FMAs on BF16 pairs with an FP32
// accumulator (PTX mixed-precision fma.rn.f32.bf16: the product of two BF16
// values is exact, one rounding per FMA, as with the FP32 FMA of the
// converted values, minus the conversions).
__device__ __forceinline__ float fma2_bf16(uint32_t w2, uint32_t x2, float acc) {
    float d;
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t.reg .f32 t;\n\t"
        "mov.b32 {wl, wh}, %1;\n\tmov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 t, wl, xl, %3;\n\tfma.rn.f32.bf16 %0, wh, xh, t;\n\t}"
        : "=f"(d)
        : "r"(w2), "r"(x2), "f"(acc));
    return d;
}

// The same from activations staged in shared memory: the lane's four 16-byte
// chunks sit at xq[(i + rot) & 3] (see stage_activations).
__device__ __forceinline__ float dot32_staged(const uint32_t (&v)[16], const uint4 *xq, uint32_t rot, float acc) {
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint4 q = xq[(i + rot) & 3u];
        acc = fma2_bf16(v[4 * i + 0], q.x, acc);
        acc = fma2_bf16(v[4 * i + 1], q.y, acc);
        acc = fma2_bf16(v[4 * i + 2], q.z, acc);
        acc = fma2_bf16(v[4 * i + 3], q.w, acc);
    }
    return acc;
}

// Copy the M x cols activations (cols a multiple of 8) into shared memory so
// that lane l's chunk i (16 bytes: columns 32 l + 8 i .. + 8 of window q) of
// row m lands in 16-byte slot (m nwin + q) 128 + 4 l + ((i + l / 2) & 3):
// the 8 lanes of each quarter-warp then read 8 different bank groups, and the
// copy's consecutive chunks write 8 different ones too. Read straight from
// global memory, each lane's 64 contiguous bytes would span 16 cache lines per
// warp-wide load (64-byte lane stride).
__device__ __forceinline__ void stage_activations(const uint16_t *x, uint32_t M, uint32_t cols, uint32_t nwin,
                                                  uint4 *dst) {
    const uint32_t cpr = cols / 8;   // 16-byte chunks per activation row
    const uint4 *src = reinterpret_cast<const uint4 *>(x);
    for (uint32_t g = threadIdx.x; g < M * cpr; g += blockDim.x) {
        const uint32_t m = g / cpr, c = g - m * cpr;
        const uint32_t q = c >> 7, l = (c & 127u) >> 2, i = c & 3u;
        dst[(m * nwin + q) * 128u + 4u * l + ((i + (l >> 1)) & 3u)] = __ldg(src + g);
    }
}

// acc + dot(v, x[0..31]) as one FMA chain; v holds the 32 weights as BF16
// pairs, x is 16-byte aligned.
__device__ __forceinline__ float dot32(const uint32_t (&v)[16], const uint16_t *x, float acc) {
    const uint4 *xp = reinterpret_cast<const uint4 *>(x);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const uint4 q = __ldg(xp + i);
        acc = fma2_bf16(v[4 * i + 0], q.x, acc);
        acc = fma2_bf16(v[4 * i + 1], q.y, acc);
        acc = fma2_bf16(v[4 * i + 2], q.z, acc);
        acc = fma2_bf16(v[4 * i + 3], q.w, acc);
    }
    return acc;
}

// Lane 0 of the warp stores the butterfly sums of acc[m] as y[m, row]; acc is reset.
template <int MM>
__device__ __forceinline__ void finish_row(float (&acc)[MM], uint32_t M, float *y, uint64_t rows, uint64_t row,
                                           uint32_t lane) {
#pragma unroll
    for (int m = 0; m < MM; m++) {
        if ((uint32_t)m < M) {
            float v = acc[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
            if (lane == 0) y[(uint64_t)m * rows + row] = v;
        }
        acc[m] = 0.f;
    }
}

// MM: the largest number of activation rows the instance handles (1, 2, 4, 8).
template <int K, int MM>
__global__ void __launch_bounds__(kLinWarps * 32, K == 16 ? 1 : K >= 14 ? 2 : 3)
    cb_linear_kernel(const __grid_constant__ CbLinBatch B) {
    using Lay = CbLinLayout<K>;
    constexpr uint32_t kWarps = Lay::kWarps;
    constexpr uint32_t kBufWords = Lay::kBufBytes / 4;
    extern __shared__ __align__(16) uint8_t smem[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Lay::kBars);
    uint32_t *bufs = reinterpret_cast<uint32_t *>(smem + Lay::kBufs);
    uint16_t *tab = reinterpret_cast<uint16_t *>(smem + Lay::kTab);
    uint4 *xst = reinterpret_cast<uint4 *>(smem + Lay::kTotal);
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const uint32_t M = B.M;

    const uint64_t r_begin = row_at_window(B, B.total_wins * blockIdx.x / gridDim.x);
    const uint64_t r_end = row_at_window(B, B.total_wins * (blockIdx.x + 1) / gridDim.x);
    if (r_begin >= r_end) return;

    uint64_t *tab_bar = &bars[2 * kWarps];
    uint64_t *my_bar = &bars[2 * warp];
    uint32_t *my_buf = bufs + 2 * warp * kBufWords;
    if (tid == 0) {
        for (uint32_t i = 0; i < 2 * kWarps + 1; i++) dev::mbar_init(&bars[i], 1);
        dev::fence_mbar_init();
    }
    __syncthreads();

    uint32_t it = 0, tab_uses = 0, status = 0;
    bool dead = false;
    uint32_t ti = 0;
    uint64_t r = r_begin;
    float acc[MM];
#pragma unroll
    for (int m = 0; m < MM; m++) acc[m] = 0.f;
    while (r < r_end) {
        while (ti + 1 < B.count && r >= B.t[ti + 1].first_row) ++ti;
        const CbLinTensor &tn = B.t[ti];
        const uint64_t seg_end = ti + 1 < B.count ? min(r_end, B.t[ti + 1].first_row) : r_end;
        const uint64_t s0 = r - tn.first_row, ns = seg_end - r;   // this tensor's rows [s0, s0 + ns)
        const uint32_t nwin = (tn.cols + kTile - 1) / kTile;
        const bool vec = (tn.cols & 7u) == 0;                    // 16-byte aligned activation chunks

        __syncthreads();
        if (tid == 0) {
            dev::fence_proxy_async_smem();
            dev::mbar_arrive_expect_tx(tab_bar, tn.table_bytes);
            dev::bulk_g2s(tab, tn.table, tn.table_bytes, tab_bar);
        }
        // this warp's (row, window) items: rows s0 + warp, + kWarps, ...; windows 0 .. nwin - 1.
        // (ir, iq): the next item to issue; (cr, cq): the item being consumed.
        uint64_t ir = s0 + warp, cr = ir;
        uint32_t iq = 0, cq = 0, issued = 0;
        const uint64_t row_end = s0 + ns;
        for (; issued < 2 && ir < row_end; issued++) {   // the first two items
            if (lane == 0 && !dead) {
                dev::fence_proxy_async_smem();   // this warp's reads of the buffer come before the copy's writes
                issue_window<K>(tn, ir, iq, my_buf + ((it + issued) & 1u) * kBufWords, &my_bar[(it + issued) & 1u]);
            }
            if (++iq == nwin) { iq = 0; ir += kWarps; }
        }
        if (tn.stage_x) stage_activations(tn.x, M, tn.cols, nwin, xst);
        const bool tab_ok = dev::mbar_wait_bounded(tab_bar, tab_uses & 1u);
        tab_uses++;
        if (__syncthreads_or(!tab_ok)) {   // also publishes the staged activations
            // let the table copy and this warp's copies land (bounded), then stop
            status |= LWC_DEVICE_TIMEOUT;
            if (tid == 0) dev::mbar_wait_bounded(tab_bar, (tab_uses - 1) & 1u);
            if (!dead)
                for (uint32_t k = 0; k < issued; k++) dev::mbar_wait_bounded(&my_bar[(it + k) & 1u], ((it + k) >> 1) & 1u);
            break;
        }

        while (cr < row_end && !dead) {
            const uint32_t bi = it & 1u;
            const bool ok = dev::mbar_wait_bounded(&my_bar[bi], (it >> 1) & 1u);
            if (__any_sync(0xFFFFFFFFu, !ok)) {
                // let this window's copy and the one issued into the other buffer land (bounded), then stop
                status |= LWC_DEVICE_TIMEOUT;
                dev::mbar_wait_bounded(&my_bar[bi], (it >> 1) & 1u);
                if (cq + 1 < nwin || cr + kWarps < row_end) dev::mbar_wait_bounded(&my_bar[bi ^ 1u], ((it + 1) >> 1) & 1u);
                dead = true;
                break;
            }
            const uint64_t bit0 = window_first(tn, cr, cq) * K;
            const uint32_t boff = (uint32_t)(bit0 - (((bit0 >> 3) & ~15ull) << 3));   // < 128
            const uint32_t cnt = window_count(tn, cq);
            const uint32_t *src = my_buf + bi * kBufWords + (boff >> 5) + lane * K;
            const uint32_t sh = boff & 31u;
            uint32_t w[K + 1];
#pragma unroll
            for (int i = 0; i < K; i++) w[i] = __funnelshift_r(src[i], src[i + 1], sh);
            w[K] = 0;
            uint32_t v[16];   // weights 2i, 2i + 1 as a BF16 pair
            Gather<K, 0>::run(w, tab, v);
            __syncwarp();
            if (lane == 0 && ir < row_end) {
                dev::fence_proxy_async_smem();
                issue_window<K>(tn, ir, iq, my_buf + bi * kBufWords, &my_bar[bi]);
            }
            if (ir < row_end && ++iq == nwin) { iq = 0; ir += kWarps; }

            const uint32_t c0 = cq * kTile + lane * 32u;
            const uint32_t valid = cnt > lane * 32u ? min(32u, cnt - lane * 32u) : 0u;
            const uint16_t *xr = tn.x + c0;
            // each window's products form their own FMA chain, then join the row's sum
            if (valid == 32u && tn.stage_x) {
                const uint4 *xq = xst + cq * 128u + 4u * lane;
#pragma unroll
                for (int m = 0; m < MM; m++)
                    if ((uint32_t)m < M) acc[m] += dot32_staged(v, xq + m * nwin * 128u, lane >> 1, 0.f);
            } else if (valid == 32u && vec) {
#pragma unroll
                for (int m = 0; m < MM; m++)
                    if ((uint32_t)m < M) acc[m] += dot32(v, xr + (uint64_t)m * tn.cols, 0.f);
            } else if (valid) {
#pragma unroll
                for (int m = 0; m < MM; m++) {
                    if ((uint32_t)m < M) {
                        const uint16_t *xm = xr + (uint64_t)m * tn.cols;
                        float p = 0.f;
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if ((uint32_t)j < valid)
                                p = fmaf(bf16_lo(v[j / 2] >> (16 * (j & 1))), bf16_lo(xm[j]), p);
                        acc[m] += p;
                    }
                }
            }
            if (++cq == nwin) {
                finish_row<MM>(acc, M, tn.y, tn.rows, cr, lane);
                cq = 0;
                cr += kWarps;
            }
            ++it;
        }
        r = seg_end;
    }
    if (status && lane == 0 && B.status) atomicOr(B.status, status);
}

// U == 1: every weight is table[0]; one warp per row, lane-strided columns
// (summation tree height ceil(cols / 32) + 5).
__global__ void cb_linear_fill_kernel(const uint16_t *__restrict__ table, const uint16_t *__restrict__ x, uint32_t M,
                                      uint64_t rows, uint32_t cols, float *__restrict__ y) {
    const float wv = __uint_as_float((uint32_t)table[0] << 16);
    const uint32_t lane = threadIdx.x & 31u;
    const uint64_t warps = (uint64_t)gridDim.x * (blockDim.x / 32);
    float acc[kMaxRows];
#pragma unroll
    for (int m = 0; m < kMaxRows; m++) acc[m] = 0.f;
    for (uint64_t r = blockIdx.x * (uint64_t)(blockDim.x / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
#pragma unroll
        for (int m = 0; m < kMaxRows; m++)
            if ((uint32_t)m < M)
                for (uint32_t c = lane; c < cols; c += 32u) acc[m] = fmaf(wv, bf16_lo(x[(uint64_t)m * cols + c]), acc[m]);
        finish_row<kMaxRows>(acc, M, y, rows, r, lane);
    }
}

// Self-test of the bounded wait the kernels use on their asynchronous copies:
// one thread waits on an mbarrier phase that completes only through its own
// arrival (`arrive`), for at most `polls` polls; a wait that gives up reports
// LWC_DEVICE_TIMEOUT and the kernel returns normally.
__global__ void wait_selftest_kernel(uint32_t *status, uint32_t polls, uint32_t arrive) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        dev::mbar_init(&bar, 1);
        if (arrive) dev::mbar_arrive(&bar);
        if (!dev::mbar_wait_bounded(&bar, 0, polls)) atomicOr(status, LWC_DEVICE_TIMEOUT);
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

using LinKernelFn = void (*)(CbLinBatch);
template <int MM>
struct LinTable {
    static constexpr LinKernelFn k[17] = {
        nullptr,                  cb_linear_kernel<1, MM>,  cb_linear_kernel<2, MM>,  cb_linear_kernel<3, MM>,
        cb_linear_kernel<4, MM>,  cb_linear_kernel<5, MM>,  cb_linear_kernel<6, MM>,  cb_linear_kernel<7, MM>,
        cb_linear_kernel<8, MM>,  cb_linear_kernel<9, MM>,  cb_linear_kernel<10, MM>, cb_linear_kernel<11, MM>,
        cb_linear_kernel<12, MM>, cb_linear_kernel<13, MM>, cb_linear_kernel<14, MM>, cb_linear_kernel<15, MM>,
        cb_linear_kernel<16, MM>};
};
constexpr int kMmCount = 4;   // instances for M <= 1, 2, 4, 8
constexpr int mm_index(uint32_t M) { return M <= 1 ? 0 : M <= 2 ? 1 : M <= 4 ? 2 : 3; }
const LinKernelFn *const kLinKernels[kMmCount] = {LinTable<1>::k, LinTable<2>::k, LinTable<4>::k, LinTable<8>::k};
template <int K>
constexpr uint32_t lin_smem_for() { return CbLinLayout<K>::kTotal; }
const uint32_t kLinSmem[17] = {0,
                               lin_smem_for<1>(),  lin_smem_for<2>(),  lin_smem_for<3>(),  lin_smem_for<4>(),
                               lin_smem_for<5>(),  lin_smem_for<6>(),  lin_smem_for<7>(),  lin_smem_for<8>(),
                               lin_smem_for<9>(),  lin_smem_for<10>(), lin_smem_for<11>(), lin_smem_for<12>(),
                               lin_smem_for<13>(), lin_smem_for<14>(), lin_smem_for<15>(), lin_smem_for<16>()};

struct DevState {
    int sms = 0;
    int per_sm[17] = {0};
    int lin_per_sm[4][17] = {{0}};
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
            for (int mi = 0; mi < kMmCount && err == cudaSuccess; mi++) {
                const void *lf = (const void *)kLinKernels[mi][k];
                err = cudaFuncSetAttribute(lf, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)(kLinSmem[k] + kXStageMax));
                if (err == cudaSuccess)
                    err = cudaFuncSetAttribute(lf, cudaFuncAttributePreferredSharedMemoryCarveout,
                                               cudaSharedmemCarveoutMaxShared);
                if (err == cudaSuccess)
                    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&s.lin_per_sm[mi][k], lf, 32 * kLinWarps,
                                                                        kLinSmem[k]);
            }
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

lwc_status launch_cb_linear_group(const std::vector<int> &idx, const lwc_desc *descs, const void *const *d_blobs,
                                  const uint64_t *cols, const uint16_t *const *d_xs, uint32_t M, float *const *d_ys,
                                  uint32_t *d_status, cudaStream_t stream, const DevState &ds) {
    CbLinBatch B;
    std::memset(&B, 0, sizeof B);
    const uint32_t K = descs[idx[0]].k;
    uint64_t rows = 0, wins = 0, xstage = 0;
    for (size_t j = 0; j < idx.size(); j++) {
        const int i = idx[j];
        const lwc_desc &d = descs[i];
        const uint8_t *base = static_cast<const uint8_t *>(d_blobs[i]);
        CbLinTensor &t = B.t[j];
        t.packed = base + d.off_packed;
        t.packed_bytes = d.packed_bytes;
        t.table = reinterpret_cast<const uint16_t *>(base + d.off_table);
        t.table_bytes = (uint32_t)((2ull * d.U + 15) / 16 * 16);
        t.x = d_xs[i];
        t.y = d_ys[i];
        t.cols = (uint32_t)cols[i];
        t.rows = d.n / cols[i];
        t.first_row = rows;
        t.first_win = wins;
        rows += t.rows;
        const uint32_t nwin = (t.cols + kTile - 1) / kTile;
        wins += t.rows * nwin;
        const uint64_t xbytes = (uint64_t)M * nwin * kTile * 2;   // whole windows
        if (t.cols % 8 == 0 && xbytes <= kXStageMax) {
            t.stage_x = 1;
            xstage = std::max<uint64_t>(xstage, xbytes);
        }
    }
    B.count = (uint32_t)idx.size();
    B.M = M;
    B.total_rows = rows;
    B.total_wins = wins;
    B.x_stage_bytes = (uint32_t)xstage;
    B.status = d_status;
    const int mi = mm_index(M);
    const size_t smem = kLinSmem[K] + xstage;
    int per_sm = ds.lin_per_sm[mi][K];
    if (xstage) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void *)kLinKernels[mi][K],
                                                                      32 * kLinWarps, smem);
        if (e != cudaSuccess) return fail(LWC_ERR_CUDA, "occupancy: %s", cudaGetErrorString(e));
    }
    per_sm = std::max(1, per_sm);
    const uint64_t grid = std::min<uint64_t>((rows + kLinWarps - 1) / kLinWarps, (uint64_t)per_sm * ds.sms);
    kLinKernels[mi][K]<<<(unsigned)grid, 32 * kLinWarps, smem, stream>>>(B);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "linear launch: %s", cudaGetErrorString(err));
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
    // one-entry tables: a fill; tables of all 65536 patterns: a copy; the rest
    // grouped by index width
    std::vector<std::vector<int>> by_k(17);
    for (int i = 0; i < count; i++) {
        const lwc_desc &d = descs[i];
        if (d.n == 0) continue;
        if (d.U == 65536) {
            const uint64_t blocks = std::min<uint64_t>((d.n + 32 * 256 - 1) / (32 * 256), (uint64_t)ds.sms * 8);
            const uint8_t *base = static_cast<const uint8_t *>(d_ins[i]);
            cb_identity_kernel<<<(unsigned)std::max<uint64_t>(blocks, 1), 256, 0, s>>>(
                base + d.off_packed, d_outs[i], d.n, reinterpret_cast<const uint16_t *>(base + d.off_table), d_status);
            cudaError_t err = cudaGetLastError();
            if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
            continue;
        }
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

lwc_status lwc_linear_codebook_batched(const lwc_desc *descs, const void *const *d_blobs, const uint64_t *cols,
                                       const uint16_t *const *d_xs, int M, float *const *d_ys, int count,
                                       uint32_t *d_status, lwc_stream_t stream) {
    if (count < 0 || (count > 0 && (!descs || !d_blobs || !cols || !d_xs || !d_ys)))
        return fail(LWC_ERR_INVALID_ARG, "bad batch arguments");
    if (M < 1 || M > kMaxRows) return fail(LWC_ERR_INVALID_ARG, "M must be 1..%d (got %d)", kMaxRows, M);
    bool any = false;
    for (int i = 0; i < count; i++) {
        lwc_status st = check_codebook_desc(&descs[i]);
        if (st) return st;
        if (cols[i] == 0 || cols[i] >= (1ull << 31) || descs[i].n % cols[i] != 0)
            return fail(LWC_ERR_INVALID_ARG, "cols must be 1..2^31-1 and divide n (tensor %d)", i);
        if (descs[i].n == 0) continue;
        any = true;
        if (!d_blobs[i] || !d_xs[i] || !d_ys[i]) return fail(LWC_ERR_INVALID_ARG, "NULL device pointer (tensor %d)", i);
        if (!aligned16(d_blobs[i]) || !aligned16(d_xs[i]) || (reinterpret_cast<uintptr_t>(d_ys[i]) & 3u))
            return fail(LWC_ERR_MISALIGNED, "blob and x must be 16-byte aligned, y 4-byte aligned (tensor %d)", i);
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
    std::vector<std::vector<int>> by_k(17);
    for (int i = 0; i < count; i++) {
        const lwc_desc &d = descs[i];
        if (d.n == 0) continue;
        if (d.k == 0) {
            const uint64_t rows = d.n / cols[i];
            const uint64_t blocks = std::min<uint64_t>((rows + 7) / 8, (uint64_t)ds.sms * 8);
            cb_linear_fill_kernel<<<(unsigned)blocks, 256, 0, s>>>(
                reinterpret_cast<const uint16_t *>(static_cast<const uint8_t *>(d_blobs[i]) + d.off_table), d_xs[i],
                (uint32_t)M, rows, (uint32_t)cols[i], d_ys[i]);
            cudaError_t err = cudaGetLastError();
            if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "linear launch: %s", cudaGetErrorString(err));
            continue;
        }
        by_k[d.k].push_back(i);
    }
    for (int k = 1; k <= 16; k++) {
        for (size_t a = 0; a < by_k[k].size(); a += kMaxBatch) {
            std::vector<int> g(by_k[k].begin() + a, by_k[k].begin() + std::min(by_k[k].size(), a + kMaxBatch));
            st = launch_cb_linear_group(g, descs, d_blobs, cols, d_xs, (uint32_t)M, d_ys, d_status, s, ds);
            if (st) return st;
        }
    }
    clear_error();
    return LWC_OK;
}

lwc_status lwc_linear_codebook(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x, int M,
                               float *d_y, uint32_t *d_status, lwc_stream_t stream) {
    if (!desc) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    return lwc_linear_codebook_batched(desc, &d_blob, &cols, &d_x, M, &d_y, 1, d_status, stream);
}

lwc_status lwc_selftest_bounded_wait(uint32_t *d_status, uint32_t polls, int arrive, lwc_stream_t stream) {
    if (!d_status || (reinterpret_cast<uintptr_t>(d_status) & 3u))
        return fail(LWC_ERR_INVALID_ARG, "status word must be a 4-byte aligned device pointer");
    if (polls == 0 || polls > (1u << 24)) return fail(LWC_ERR_INVALID_ARG, "polls must be 1..2^24");
    wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(d_status, polls, arrive ? 1u : 0u);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(err));
    clear_error();
    return LWC_OK;
}

}  // extern "C"
