// Device-side encoders: the same blobs as the host encoders (byte for byte),
// built from a tensor that is already in GPU memory, so that a model loaded
// in BF16 onto the GPU can be compressed there without a round trip through
// host memory.
//
// The motivation is the load-time cost that "Codebook Lossless Compression:
// когда 25% памяти значат больше, чем кажется" (ai-manual.ru, section on
// the trade-offs) reports: setting up the dictionary and the index map makes
// loading slower. Here every pass over the weights runs on the GPU; only the
// small decisions (the Huffman code from a 256-bin histogram, the codebook
// table from a 65536-bit presence map) are taken on the host, by the same
// code the host encoders use, so both produce identical blobs.
//
// DFloat11 ("Koniec z kompromisami! DFloat11 ratuje dokładność modeli AI
// ...", section "Przełom: DFloat11"): exponent histogram on the device; code
// lengths, canonical codes and lookup tables on the host; then on the device
// the bit length of every 4096-weight tile, a scan of those lengths into tile
// start bits, and one pass that writes each tile's codes (assembled in shared
// memory), the per-chunk gaps, the per-block output offsets and the
// sign|mantissa bytes; a last pass finds the largest block.
//
// Codebook ("Как работает эта магия?" on the page above): presence bitmap on
// the device, sorted table and index map on the host, then one packing pass.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "lwc_internal.h"

namespace lwc {
namespace {

// ---------------------------------------------------------------- workspace

constexpr uint32_t kWsMagic = 0x4B57434Cu;       // a plan is stored in the workspace
constexpr uint64_t kWsCounts = 256;              // u64[256] histogram or u32[2048] presence bitmap
constexpr uint64_t kWsArrays = kWsCounts + 8192;  // tile arrays (DFloat11) or u16[65536] index map
constexpr uint64_t kMaxDeviceN = 1ull << 36;     // per-CTA shared counters stay below 2^32

constexpr uint32_t kTile = 4096;        // weights per tile of the DFloat11 passes
constexpr uint32_t kTileThreads = 256;  // 16 weights per thread
constexpr uint32_t kPerThread = kTile / kTileThreads;
constexpr uint32_t kPackWarps = 8;      // codebook packing: warps per CTA, 1024 weights per warp tile

constexpr uint32_t kErrUnplanned = 1;   // an exponent the plan has no code for
constexpr uint32_t kErrOverflow = 2;    // more bits than planned

// The workspace's first bytes: the plan's inputs (so that the write call can
// rebuild the exact same plan) and the results of the write kernels.
struct WsHeader {
    uint32_t magic;
    uint32_t codec;
    uint64_t n;
    uint32_t chunk_bytes;
    uint32_t threads_per_block;
    uint32_t max_len;
    uint32_t error;            // kErr* bits
    uint64_t total_bits;       // written by the scan
    uint32_t max_block_count;  // written by the last pass
    uint32_t elem;             // LWC_ELEM_* of the source
    uint32_t chunk_counts;     // store per-chunk code counts when they fit a byte
};
static_assert(sizeof(WsHeader) <= kWsCounts, "workspace header too large");

constexpr uint64_t n_tiles_of(uint64_t n) { return (n + kTile - 1) / kTile; }
constexpr uint64_t ws_tile_pos_off(uint64_t n) { return kWsArrays + round_up(4 * n_tiles_of(n), 256); }

constexpr uint64_t workspace_bytes(uint64_t n) {
    const uint64_t df11 = ws_tile_pos_off(n) + 8 * (n_tiles_of(n) + 1);
    const uint64_t cb = kWsArrays + 2 * 65536;
    return round_up(std::max(df11, cb), 256);
}

// (length << 32) | codeword, by exponent value; passed by value to the kernels.
struct CodeTable {
    uint64_t lc[256];
};

// ------------------------------------------------------------ device helpers

// Element i of the source as a BF16-shaped pattern (sign, exponent field, top
// 7 mantissa bits; see the element types in lwc.h), from its raw bits.
template <int E>
__device__ __forceinline__ uint32_t shaped(uint32_t x) {
    if constexpr (E == LWC_ELEM_FP32) return x >> 16;
    else if constexpr (E == LWC_ELEM_FP16) return (x & 0x8000u) | ((x >> 3) & 0x0FFFu);
    else return x;
}

// Two 16-bit elements packed in a word (low half first), each made BF16-shaped.
template <int E>
__device__ __forceinline__ uint32_t shaped_pair(uint32_t w) {
    if constexpr (E == LWC_ELEM_FP16) return (w & 0x80008000u) | ((w >> 3) & 0x0FFF0FFFu);
    else return w;
}

// Loads elements i0 .. i0+15 as 8 words of BF16-shaped patterns (two per
// word, low half first); elements at or past n read as 0. Returns how many
// are below n. The source holds uint32 elements for FP32, uint16 otherwise.
template <int E>
__device__ __forceinline__ uint32_t load16(const void *__restrict__ src, uint64_t n, uint64_t i0, uint32_t w[8]) {
    if constexpr (E == LWC_ELEM_FP32) {
        const uint32_t *x = static_cast<const uint32_t *>(src);
        if (i0 + kPerThread <= n) {
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint4 a = __ldg(reinterpret_cast<const uint4 *>(x + i0) + q);
                w[2 * q] = __byte_perm(a.x, a.y, 0x7632u);       // high halves of two elements
                w[2 * q + 1] = __byte_perm(a.z, a.w, 0x7632u);
            }
            return kPerThread;
        }
#pragma unroll
        for (int j = 0; j < 8; j++) w[j] = 0;
        if (i0 >= n) return 0;
        const uint32_t cnt = (uint32_t)(n - i0);
#pragma unroll
        for (uint32_t k = 0; k < kPerThread; k++)
            if (k < cnt) w[k >> 1] |= (x[i0 + k] >> 16) << (16 * (k & 1));
        return cnt;
    } else {
        const uint16_t *x = static_cast<const uint16_t *>(src);
        if (i0 + kPerThread <= n) {
            const uint4 a = __ldg(reinterpret_cast<const uint4 *>(x + i0));
            const uint4 b = __ldg(reinterpret_cast<const uint4 *>(x + i0) + 1);
            w[0] = a.x, w[1] = a.y, w[2] = a.z, w[3] = a.w, w[4] = b.x, w[5] = b.y, w[6] = b.z, w[7] = b.w;
#pragma unroll
            for (int j = 0; j < 8; j++) w[j] = shaped_pair<E>(w[j]);
            return kPerThread;
        }
#pragma unroll
        for (int j = 0; j < 8; j++) w[j] = 0;
        if (i0 >= n) return 0;
        const uint32_t cnt = (uint32_t)(n - i0);
#pragma unroll
        for (uint32_t k = 0; k < kPerThread; k++)
            if (k < cnt) w[k >> 1] |= shaped<E>(x[i0 + k]) << (16 * (k & 1));
        return cnt;
    }
}

__device__ __forceinline__ uint32_t exponent_of(const uint32_t w[8], uint32_t j) {
    return (w[j >> 1] >> (16 * (j & 1) + 7)) & 0xFF;
}

// Exclusive scan over the CTA (kTileThreads threads); *total gets the sum.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *s_warp, uint32_t *total) {
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, d);
        if (lane >= (uint32_t)d) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (uint32_t k = 0; k < kTileThreads / 32; k++) {
        const uint32_t t = s_warp[k];
        before += k < warp ? t : 0;
        all += t;
    }
    *total = all;
    return before + x - v;
}

// ------------------------------------------------------------ DFloat11 kernels

// Exponent histogram. Each lane owns one copy of the 256 counters and the
// copies are interleaved so that the 32 lanes of a warp always hit 32
// different banks, whatever exponents they see (weights cluster on a few
// exponent values, which would serialise a single shared histogram).
template <int E>
__global__ void __launch_bounds__(512) df11_histogram_kernel(const void *__restrict__ src, uint64_t n,
                                                             unsigned long long *counts) {
    __shared__ uint32_t h[256 * 32];
    for (uint32_t i = threadIdx.x; i < 256 * 32; i += blockDim.x) h[i] = 0;
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31;
    const uint64_t groups = (n + kPerThread - 1) / kPerThread, stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t g = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; g < groups; g += stride) {
        uint32_t w[8];
        const uint32_t cnt = load16<E>(src, n, g * kPerThread, w);
#pragma unroll
        for (uint32_t j = 0; j < kPerThread; j++)
            if (j < cnt) atomicAdd(&h[exponent_of(w, j) * 32 + lane], 1u);
    }
    __syncthreads();
    for (uint32_t e = threadIdx.x; e < 256; e += blockDim.x) {
        uint32_t sum = 0;
        for (uint32_t l = 0; l < 32; l++) sum += h[e * 32 + ((l + e) & 31)];  // rotated: no bank conflicts
        if (sum) atomicAdd(&counts[e], (unsigned long long)sum);
    }
}

// Bit length of every tile (sum of its code lengths).
template <int E>
__global__ void __launch_bounds__(kTileThreads) df11_tile_bits_kernel(const void *__restrict__ src, uint64_t n,
                                                                      uint64_t n_tiles, CodeTable t,
                                                                      uint32_t *tile_bits, WsHeader *ws) {
    __shared__ uint32_t s_len[256];
    __shared__ uint32_t s_warp[kTileThreads / 32];
    s_len[threadIdx.x] = (uint32_t)(t.lc[threadIdx.x] >> 32);
    __syncthreads();
    bool bad = false;
    for (uint64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        uint32_t w[8];
        const uint32_t cnt = load16<E>(src, n, tile * kTile + threadIdx.x * kPerThread, w);
        uint32_t bits = 0;
#pragma unroll
        for (uint32_t j = 0; j < kPerThread; j++) {
            if (j < cnt) {
                const uint32_t l = s_len[exponent_of(w, j)];
                bits += l;
                bad |= l == 0;
            }
        }
        uint32_t total;
        block_exclusive_scan(bits, s_warp, &total);
        if (threadIdx.x == 0) tile_bits[tile] = total;
        __syncthreads();
    }
    if (bad) atomicOr(&ws->error, kErrUnplanned);
}

// Exclusive scan of the tile lengths into tile start bits (one CTA). Also
// zeroes every stream word that two tiles share (a tile starting inside a
// word), which the emit pass then fills with atomicOr from both sides.
__global__ void __launch_bounds__(1024) df11_scan_kernel(const uint32_t *tile_bits, uint64_t *tile_pos,
                                                         uint64_t n_tiles, uint32_t *stream, uint64_t stream_words,
                                                         WsHeader *ws) {
    __shared__ unsigned long long s_warp[32];
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint64_t per = (n_tiles + blockDim.x - 1) / blockDim.x;
    const uint64_t b = std::min<uint64_t>(n_tiles, threadIdx.x * per), e = std::min<uint64_t>(n_tiles, b + per);
    unsigned long long sum = 0;
    for (uint64_t i = b; i < e; i++) sum += tile_bits[i];
    unsigned long long x = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, x, d);
        if (lane >= (uint32_t)d) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    unsigned long long run = x - sum;
    for (uint32_t k = 0; k < warp; k++) run += s_warp[k];
    for (uint64_t i = b; i < e; i++) {
        tile_pos[i] = run;
        if ((run & 31) && (run >> 5) < stream_words) stream[run >> 5] = 0;
        run += tile_bits[i];
    }
    if (threadIdx.x == blockDim.x - 1) {
        tile_pos[n_tiles] = run;
        ws->total_bits = run;
    }
}

struct EmitArgs {
    const void *src;
    uint64_t n;
    const uint64_t *tile_pos;
    uint64_t n_tiles;
    uint32_t *stream;
    uint64_t stream_words;  // words that hold code bits: ceil(total_bits / 32)
    uint8_t *gaps;
    uint32_t *counts;       // per-chunk code counts as bytes of u32 words (zeroed first), or null
    uint64_t n_chunks;
    uint64_t chunk_bits;
    uint64_t *blkoff;
    uint64_t n_blocks;
    uint64_t block_bits;
    uint8_t *sm;
    WsHeader *ws;
};

// Sign|mantissa byte of the BF16 pattern in the low (hi = 0) or high half of w.
__device__ __forceinline__ uint32_t sm_byte(uint32_t w, int hi) {
    const uint32_t x = w >> (16 * hi);
    return ((x >> 8) & 0x80) | (x & 0x7F);
}

// Writes one tile per iteration: codes MSB-first into a shared-memory copy
// of the tile's stream words, then the words out (atomicOr on the two words a
// tile may share with its neighbours, plain stores elsewhere). A code that
// crosses a chunk start gives that chunk's gap (bits from the chunk start to
// the next code); one that crosses a block start gives that block's first
// weight index. Codes are at most 32 bits and chunks at least 64, so a code
// crosses at most one chunk start. With per-chunk code counts, each thread
// counts its codes per chunk and adds each chunk's part to that chunk's byte
// (an atomic add on the byte's word: the plan guarantees that no chunk holds
// more than 255 codes, so no carry reaches the next byte).
template <int E>
__global__ void __launch_bounds__(kTileThreads) df11_emit_kernel(EmitArgs a, CodeTable t) {
    __shared__ uint64_t s_lc[256];
    __shared__ uint32_t s_words[kTile + 2];  // 32 bits per weight at most, plus the lead-in word
    __shared__ uint32_t s_warp[kTileThreads / 32];
    __shared__ uint64_t s_div[4];            // tile start bit / and % chunk bits, / and % block bits
    s_lc[threadIdx.x] = t.lc[threadIdx.x];
    __syncthreads();
    const uint64_t n16 = (a.n + 15) & ~15ull;
    uint32_t err = 0;
    for (uint64_t tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
        const uint64_t i0 = tile * kTile + threadIdx.x * kPerThread;
        uint32_t w[8];
        const uint32_t cnt = load16<E>(a.src, a.n, i0, w);
        if (i0 < n16) {
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; k++)
                o[k] = sm_byte(w[2 * k], 0) | sm_byte(w[2 * k], 1) << 8 | sm_byte(w[2 * k + 1], 0) << 16 |
                       sm_byte(w[2 * k + 1], 1) << 24;
            *reinterpret_cast<uint4 *>(a.sm + i0) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        uint32_t bits = 0;
#pragma unroll
        for (uint32_t j = 0; j < kPerThread; j++)
            if (j < cnt) bits += (uint32_t)(s_lc[exponent_of(w, j)] >> 32);
        uint32_t tile_bits;
        const uint32_t excl = block_exclusive_scan(bits, s_warp, &tile_bits);
        const uint64_t t0 = a.tile_pos[tile];
        const uint32_t lead = (uint32_t)(t0 & 31);
        const uint32_t nwords = (lead + tile_bits + 31) / 32;
        for (uint32_t j = threadIdx.x; j < nwords; j += kTileThreads) s_words[j] = 0;
        if (threadIdx.x == 0) {   // the tile's 64-bit divisions, once
            s_div[0] = t0 / a.chunk_bits;
            s_div[1] = t0 % a.chunk_bits;
            s_div[2] = t0 / a.block_bits;
            s_div[3] = t0 % a.block_bits;
        }
        __syncthreads();

        if (cnt) {
            if (i0 == 0) {
                a.gaps[0] = 0;
                a.blkoff[0] = 0;
            }
            const uint32_t o0 = lead + excl;
            // chunk and block starts after this thread's first code, as 32-bit
            // distances from it (chunks are <= 8192 bits, blocks <= 2^23)
            const uint32_t cbits = (uint32_t)a.chunk_bits, bbits = (uint32_t)a.block_bits;
            const uint32_t xc = (uint32_t)s_div[1] + excl, xb = (uint32_t)s_div[3] + excl;
            uint64_t ci = s_div[0] + xc / cbits + 1, bi = s_div[2] + xb / bbits + 1;
            uint32_t next_c = cbits - xc % cbits, next_b = bbits - xb % bbits, rel = 0;
            uint64_t acc = 0;
            uint32_t nacc = o0 & 31, wi = o0 >> 5, run = 0;
            bool first = true;
            // adds this thread's run of codes to the count of chunk ci - 1, where they start
            auto flush = [&]() {
                if (a.counts && run && ci - 1 < a.n_chunks)
                    atomicAdd(&a.counts[(ci - 1) >> 2], run << (8u * (uint32_t)((ci - 1) & 3)));
                run = 0;
            };
#pragma unroll
            for (uint32_t j = 0; j < kPerThread; j++) {
                if (j >= cnt) break;
                const uint64_t lc = s_lc[exponent_of(w, j)];
                const uint32_t l = (uint32_t)(lc >> 32);
                if (l == 0) {
                    err |= kErrUnplanned;
                    continue;
                }
                acc = (acc << l) | (uint32_t)lc;
                nacc += l;
                if (nacc >= 32) {
                    nacc -= 32;
                    const uint32_t word = (uint32_t)(acc >> nacc);
                    if (first) atomicOr(&s_words[wi], word);  // shares bits with the previous thread
                    else s_words[wi] = word;
                    wi++;
                    first = false;
                }
                const uint32_t end = rel + l;
                run++;
                if (end >= next_c) {
                    if (ci < a.n_chunks) a.gaps[ci] = (uint8_t)(end - next_c);
                    flush();
                    ci++;
                    next_c += cbits;
                }
                if (end >= next_b) {
                    if (bi < a.n_blocks) a.blkoff[bi] = i0 + j + 1;
                    bi++;
                    next_b += bbits;
                }
                rel = end;
            }
            if (nacc) atomicOr(&s_words[wi], (uint32_t)(acc << (32 - nacc)));
            flush();
            if (i0 + cnt == a.n) a.blkoff[a.n_blocks] = a.n;
        }
        __syncthreads();

        const uint64_t w0 = t0 >> 5, t_end = t0 + tile_bits;
        const bool last = tile + 1 == a.n_tiles;
        for (uint32_t j = threadIdx.x; j < nwords; j += kTileThreads) {
            const uint64_t gw = w0 + j;
            if (gw >= a.stream_words) {
                err |= kErrOverflow;
                continue;
            }
            const bool shared = (j == 0 && lead) || (j == nwords - 1 && (t_end & 31) && !last);
            if (shared) atomicOr(&a.stream[gw], s_words[j]);
            else a.stream[gw] = s_words[j];
        }
        __syncthreads();
    }
    if (err) atomicOr(&a.ws->error, err);
}

// Sign|mantissa bytes only (tensors with a single exponent value: no stream).
template <int E>
__global__ void __launch_bounds__(kTileThreads) df11_sm_kernel(const void *__restrict__ src, uint64_t n,
                                                               uint8_t *sm) {
    const uint64_t n16 = (n + 15) & ~15ull;
    for (uint64_t i0 = ((uint64_t)blockIdx.x * kTileThreads + threadIdx.x) * kPerThread; i0 < n16;
         i0 += (uint64_t)gridDim.x * kTileThreads * kPerThread) {
        uint32_t w[8];
        load16<E>(src, n, i0, w);
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; k++)
            o[k] = sm_byte(w[2 * k], 0) | sm_byte(w[2 * k], 1) << 8 | sm_byte(w[2 * k + 1], 0) << 16 |
                   sm_byte(w[2 * k + 1], 1) << 24;
        *reinterpret_cast<uint4 *>(sm + i0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// The raw low-mantissa section: FP32 low halves (uint16 per element), FP16
// low 3 mantissa bits (48 bits per 16 elements, at byte 6 (i0 / 16), least
// significant bits first). Elements past n contribute zeros.
template <int E>
__global__ void __launch_bounds__(kTileThreads) df11_lo_kernel(const void *__restrict__ src, uint64_t n, uint8_t *lo) {
    const uint64_t groups = (n + kPerThread - 1) / kPerThread;
    for (uint64_t g = (uint64_t)blockIdx.x * kTileThreads + threadIdx.x; g < groups;
         g += (uint64_t)gridDim.x * kTileThreads) {
        const uint64_t i0 = g * kPerThread;
        if constexpr (E == LWC_ELEM_FP32) {
            const uint32_t *x = static_cast<const uint32_t *>(src);
            uint16_t *o = reinterpret_cast<uint16_t *>(lo) + i0;
            if (i0 + kPerThread <= n) {
                uint32_t p[8];
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(x + i0) + q);
                    p[2 * q] = __byte_perm(a.x, a.y, 0x5410u);   // low halves of two elements
                    p[2 * q + 1] = __byte_perm(a.z, a.w, 0x5410u);
                }
                reinterpret_cast<uint4 *>(o)[0] = make_uint4(p[0], p[1], p[2], p[3]);
                reinterpret_cast<uint4 *>(o)[1] = make_uint4(p[4], p[5], p[6], p[7]);
            } else {
                for (uint64_t i = i0; i < n; i++) o[i - i0] = (uint16_t)x[i];
            }
        } else {
            const uint16_t *x = static_cast<const uint16_t *>(src);
            uint64_t bits = 0;
#pragma unroll
            for (uint32_t k = 0; k < kPerThread; k++)
                if (i0 + k < n) bits |= (uint64_t)(x[i0 + k] & 7u) << (3 * k);
            uint16_t *o = reinterpret_cast<uint16_t *>(lo + 6 * g);   // even byte: 16-bit stores
            o[0] = (uint16_t)bits;
            o[1] = (uint16_t)(bits >> 16);
            o[2] = (uint16_t)(bits >> 32);
        }
    }
}

// Largest number of weights one decoding block covers.
__global__ void __launch_bounds__(256) df11_max_block_kernel(const uint64_t *blkoff, uint64_t n_blocks, WsHeader *ws) {
    uint32_t m = 0;
    for (uint64_t b = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks; b += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t d = blkoff[b + 1] - blkoff[b];
        m = max(m, (uint32_t)(d > 0xFFFFFFFFull ? 0xFFFFFFFFull : d));
    }
#pragma unroll
    for (int d = 16; d; d >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, d));
    if ((threadIdx.x & 31) == 0 && m) atomicMax(&ws->max_block_count, m);
}

// ------------------------------------------------------------ codebook kernels

// Which of the 65536 patterns occur. A bit already set is only read, so the
// common patterns cost a shared-memory load and no atomic.
__global__ void __launch_bounds__(512) cb_presence_kernel(const uint16_t *__restrict__ src, uint64_t n,
                                                          uint32_t *bitmap) {
    __shared__ uint32_t s_bits[2048];
    for (uint32_t i = threadIdx.x; i < 2048; i += blockDim.x) s_bits[i] = 0;
    __syncthreads();
    volatile uint32_t *vb = s_bits;
    const uint64_t nv = n / 8, stride = (uint64_t)gridDim.x * blockDim.x;
    const uint4 *v = reinterpret_cast<const uint4 *>(src);
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
        const uint4 q = __ldg(v + i);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const uint32_t p = (w[j >> 1] >> (16 * (j & 1))) & 0xFFFF, m = 1u << (p & 31);
            if (!(vb[p >> 5] & m)) atomicOr(&s_bits[p >> 5], m);
        }
    }
    if (blockIdx.x == 0)
        for (uint64_t i = nv * 8 + threadIdx.x; i < n; i += blockDim.x) atomicOr(&s_bits[src[i] >> 5], 1u << (src[i] & 31));
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < 2048; i += blockDim.x)
        if (s_bits[i]) atomicOr(&bitmap[i], s_bits[i]);
}

// The ascending table of present patterns and the pattern -> index map, from
// the presence bitmap: a pattern's index is the number of set bits before it.
// 2048 threads (8 CTAs of 256), one bitmap word of 32 patterns each; a CTA
// counts the set bits of all earlier CTAs' words itself, then scans its own.
// Absent patterns map to 0xFFFF. A count that differs from the planned U is
// flagged.
constexpr uint32_t kRankCtas = 8, kRankThreads = 256;

__global__ void __launch_bounds__(kRankThreads) cb_rank_kernel(const uint32_t *bitmap, uint16_t *rank,
                                                               uint16_t *table, uint32_t U, WsHeader *ws) {
    __shared__ uint32_t s_warp[kRankThreads / 32];
    __shared__ uint32_t s_before;
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // set bits in the words of earlier CTAs
    uint32_t before = 0;
    for (uint32_t i = threadIdx.x; i < blockIdx.x * kRankThreads; i += kRankThreads) before += __popc(bitmap[i]);
#pragma unroll
    for (int d = 16; d; d >>= 1) before += __shfl_xor_sync(0xFFFFFFFFu, before, d);
    if (lane == 0) s_warp[warp] = before;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
        for (uint32_t k = 0; k < kRankThreads / 32; k++) t += s_warp[k];
        s_before = t;
    }
    __syncthreads();
    // exclusive scan of this CTA's word counts
    const uint32_t wi = blockIdx.x * kRankThreads + threadIdx.x;
    const uint32_t word = bitmap[wi], c = __popc(word);
    uint32_t x = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, d);
        if (lane >= (uint32_t)d) x += y;
    }
    if (lane == 31) s_warp[warp] = x;   // every thread has read s_warp above (second barrier)
    __syncthreads();
    uint32_t r = s_before + x - c, total = s_before;
    for (uint32_t k = 0; k < kRankThreads / 32; k++) {
        r += k < warp ? s_warp[k] : 0;
        total += s_warp[k];
    }
    uint32_t pairs[16];
#pragma unroll
    for (int b = 0; b < 32; b += 2) {
        const bool s0 = (word >> b) & 1u, s1 = (word >> (b + 1)) & 1u;
        const uint32_t r0 = s0 ? r : 0xFFFFu;
        if (s0 && r < U) table[r] = (uint16_t)(32 * wi + b);
        r += s0;
        const uint32_t r1 = s1 ? r : 0xFFFFu;
        if (s1 && r < U) table[r] = (uint16_t)(32 * wi + b + 1);
        r += s1;
        pairs[b / 2] = r0 | (r1 << 16);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(rank + 32 * wi);
#pragma unroll
    for (int q = 0; q < 4; q++) dst[q] = make_uint4(pairs[4 * q], pairs[4 * q + 1], pairs[4 * q + 2], pairs[4 * q + 3]);
    if (blockIdx.x == kRankCtas - 1 && threadIdx.x == kRankThreads - 1 && total != U) atomicOr(&ws->error, kErrUnplanned);
}

// Packs K-bit indices, LSB first. A warp handles 1024 weights: 32 lanes x 32
// consecutive weights, whose K-bit indices fill exactly K words per lane.
// Patterns are staged in shared memory (16-byte slots XOR-swizzled within
// each 128-byte row, so that both the coalesced fill and each lane's read of
// its own 64 bytes are conflict-free), and the packed words are staged again
// so that the warp stores 32 consecutive words at a time.
//
// Patterns the plan did not see map to index 0xFFFF (never a valid index when
// U < 65536, and with U = 65536 every pattern is seen); they are flagged in
// the workspace and packed as 0 so that they cannot spill into other indices.
template <int K>
__global__ void __launch_bounds__(kPackWarps * 32) cb_pack_kernel(const uint16_t *__restrict__ src, uint64_t n,
                                                                  const uint16_t *__restrict__ rank, uint32_t U,
                                                                  uint32_t *packed, uint64_t packed_words,
                                                                  WsHeader *ws) {
    __shared__ uint4 s_in[kPackWarps][128];
    __shared__ uint32_t s_out[kPackWarps][K * 33];
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint64_t groups = (n + 1023) / 1024;
    bool bad = false;
    for (uint64_t g = (uint64_t)blockIdx.x * kPackWarps + warp; g < groups; g += (uint64_t)gridDim.x * kPackWarps) {
        const uint64_t base = g * 1024;
#pragma unroll
        for (uint32_t it = 0; it < 4; it++) {
            const uint32_t u = it * 32 + lane;
            const uint64_t i = base + 8 * u;
            uint4 q;
            if (i + 8 <= n) {
                q = __ldg(reinterpret_cast<const uint4 *>(src + i));
            } else {
                uint32_t x[4] = {0, 0, 0, 0};
#pragma unroll
                for (uint32_t k = 0; k < 8; k++)
                    if (i + k < n) x[k >> 1] |= (uint32_t)src[i + k] << (16 * (k & 1));
                q = make_uint4(x[0], x[1], x[2], x[3]);
            }
            s_in[warp][u ^ ((u >> 3) & 7)] = q;
        }
        __syncwarp();
        uint32_t idx[32];
#pragma unroll
        for (uint32_t v = 0; v < 4; v++) {
            const uint32_t u = 4 * lane + v;
            const uint4 q = s_in[warp][u ^ ((u >> 3) & 7)];
            const uint32_t x[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (uint32_t h = 0; h < 8; h++) {
                const uint64_t i = base + 32 * lane + 8 * v + h;
                const uint32_t p = (x[h >> 1] >> (16 * (h & 1))) & 0xFFFF;
                uint32_t r = i < n ? __ldg(rank + p) : 0;
                bad |= r >= U;
                idx[8 * v + h] = r < U ? r : 0;
            }
        }
        uint32_t out[K];
#pragma unroll
        for (int q = 0; q < K; q++) out[q] = 0;
#pragma unroll
        for (int j = 0; j < 32; j++) {
            const int b = j * K, q = b >> 5, s = b & 31;
            out[q] |= idx[j] << s;
            if (s + K > 32) out[q + 1] |= idx[j] >> (32 - s);
        }
#pragma unroll
        for (int q = 0; q < K; q++) s_out[warp][q * 33 + lane] = out[q];
        __syncwarp();
        const uint64_t w0 = g * 32 * K;
#pragma unroll
        for (uint32_t it = 0; it < (uint32_t)K; it++) {
            const uint32_t wd = it * 32 + lane;
            const uint64_t gw = w0 + wd;
            if (gw < packed_words) packed[gw] = s_out[warp][(wd % K) * 33 + wd / K];
        }
        __syncwarp();
    }
    if (bad) atomicOr(&ws->error, kErrUnplanned);
}

typedef void (*PackKernel)(const uint16_t *, uint64_t, const uint16_t *, uint32_t, uint32_t *, uint64_t, WsHeader *);
const PackKernel kPackKernels[16] = {cb_pack_kernel<1>,  cb_pack_kernel<2>,  cb_pack_kernel<3>,  cb_pack_kernel<4>,
                                     cb_pack_kernel<5>,  cb_pack_kernel<6>,  cb_pack_kernel<7>,  cb_pack_kernel<8>,
                                     cb_pack_kernel<9>,  cb_pack_kernel<10>, cb_pack_kernel<11>, cb_pack_kernel<12>,
                                     cb_pack_kernel<13>, cb_pack_kernel<14>, cb_pack_kernel<15>, cb_pack_kernel<16>};

// ------------------------------------------------------------ host side

#define LWC_CUDA(call, what)                                                                \
    do {                                                                                    \
        cudaError_t e_ = (call);                                                            \
        if (e_ != cudaSuccess) return fail(LWC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_)); \
    } while (0)

lwc_status grid_for(const void *kernel, int threads, int smem, uint64_t work_items, unsigned &grid) {
    int dev = 0, sms = 0, per_sm = 0;
    LWC_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    LWC_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev), "device attributes");
    LWC_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem), "occupancy");
    const uint64_t full = (uint64_t)std::max(1, sms) * std::max(1, per_sm);
    grid = (unsigned)std::max<uint64_t>(1, std::min<uint64_t>(full, work_items));
    return LWC_OK;
}

lwc_status check_common(const void *d_src, uint64_t n, void *d_work, uint64_t work_bytes) {
    if (!d_work) return fail(LWC_ERR_INVALID_ARG, "NULL workspace");
    if (n && !d_src) return fail(LWC_ERR_INVALID_ARG, "NULL source");
    if (n > kMaxDeviceN) return fail(LWC_ERR_UNSUPPORTED, "tensor of %llu weights is above the device encoder's limit",
                                     (unsigned long long)n);
    if (!aligned16(d_src) || (reinterpret_cast<uintptr_t>(d_work) & 255))
        return fail(LWC_ERR_MISALIGNED, "source must be 16-byte and workspace 256-byte aligned");
    if (work_bytes < workspace_bytes(n))
        return fail(LWC_ERR_INVALID_ARG, "workspace of %llu bytes, %llu needed", (unsigned long long)work_bytes,
                    (unsigned long long)workspace_bytes(n));
    return LWC_OK;
}

lwc_status fetch_header(void *d_work, WsHeader &h, void *host, uint64_t bytes, cudaStream_t s) {
    LWC_CUDA(cudaMemcpyAsync(&h, d_work, sizeof h, cudaMemcpyDeviceToHost, s), "workspace read");
    if (host) LWC_CUDA(cudaMemcpyAsync(host, static_cast<uint8_t *>(d_work) + kWsCounts, bytes,
                                       cudaMemcpyDeviceToHost, s), "workspace read");
    LWC_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    return LWC_OK;
}

lwc_status put_header(void *d_work, const WsHeader &h, cudaStream_t s) {
    LWC_CUDA(cudaMemcpyAsync(d_work, &h, sizeof h, cudaMemcpyHostToDevice, s), "workspace write");
    return LWC_OK;
}

lwc_status zero(void *base, uint64_t from, uint64_t to, cudaStream_t s) {
    if (to > from) LWC_CUDA(cudaMemsetAsync(static_cast<uint8_t *>(base) + from, 0, to - from, s), "memset");
    return LWC_OK;
}

lwc_status finish_blob(void *d_blob, const lwc_desc &d, lwc_desc *desc_out, cudaStream_t s) {
    uint8_t header[kHeaderBytes];
    write_header(header, d);
    LWC_CUDA(cudaMemcpyAsync(d_blob, header, kHeaderBytes, cudaMemcpyHostToDevice, s), "header write");
    LWC_CUDA(cudaStreamSynchronize(s), "stream synchronize");
    *desc_out = d;
    return LWC_OK;
}

// The raw low-mantissa section of FP32 / FP16 blobs, and the zero padding after it.
template <int E>
lwc_status write_lo(const void *src, uint64_t n, uint8_t *blob, const lwc_desc &d, cudaStream_t s) {
    if constexpr (E == LWC_ELEM_BF16) {
        return LWC_OK;
    } else {
        const uint64_t groups = (n + kPerThread - 1) / kPerThread;
        const uint64_t written = E == LWC_ELEM_FP32 ? 2 * n : 6 * groups;
        if (lwc_status st = zero(blob, d.off_sm + round_up(n, 16), d.off_lo, s)) return st;   // padding before it
        if (lwc_status st = zero(blob, d.off_lo + written, d.off_lo + d.lo_bytes, s)) return st;
        if (!n) return LWC_OK;
        unsigned grid;
        if (lwc_status st = grid_for((const void *)df11_lo_kernel<E>, kTileThreads, 0,
                                     (groups + kTileThreads - 1) / kTileThreads, grid))
            return st;
        df11_lo_kernel<E><<<grid, kTileThreads, 0, s>>>(src, n, blob + d.off_lo);
        LWC_CUDA(cudaGetLastError(), "encode launch");
        return LWC_OK;
    }
}

template <int E>
lwc_status write_dfloat11(const void *src, uint64_t n, const WsHeader &h, const uint64_t *counts,
                          uint8_t *work, uint8_t *blob, uint64_t blob_bytes, lwc_desc *desc_out, cudaStream_t s) {
    Df11Plan plan;
    if (lwc_status st = plan_dfloat11(counts, n, h.chunk_bytes, h.threads_per_block, h.max_len, h.chunk_counts != 0,
                                      plan, lo_section_bytes(E, n)))
        return st;
    plan.d.elem = E;
    lwc_desc &d = plan.d;
    if (blob_bytes < d.total_bytes)
        return fail(LWC_ERR_INVALID_ARG, "blob buffer of %llu bytes, %llu needed", (unsigned long long)blob_bytes,
                    (unsigned long long)d.total_bytes);
    if (lwc_status st = write_lo<E>(src, n, blob, d, s)) return st;
    if (plan.single) {
        if (lwc_status st = zero(blob, kHeaderBytes, d.off_sm, s)) return st;
        if (n) {
            unsigned grid;
            if (lwc_status st = grid_for((const void *)df11_sm_kernel<E>, kTileThreads, 0, n_tiles_of(n), grid))
                return st;
            df11_sm_kernel<E><<<grid, kTileThreads, 0, s>>>(src, n, blob + d.off_sm);
            LWC_CUDA(cudaGetLastError(), "encode launch");
        }
        return finish_blob(blob, d, desc_out, s);
    }

    uint8_t lengths[256];
    for (int e = 0; e < 256; e++) lengths[e] = (uint8_t)plan.len[e];
    CodeTable t;
    for (int e = 0; e < 256; e++) t.lc[e] = ((uint64_t)plan.len[e] << 32) | plan.code[e];
    const uint64_t stream_words = (d.total_bits + 31) / 32, tiles = n_tiles_of(n);
    WsHeader hw = h;
    hw.error = 0;
    hw.total_bits = 0;
    hw.max_block_count = 0;
    if (lwc_status st = put_header(work, hw, s)) return st;
    LWC_CUDA(cudaMemcpyAsync(blob + d.off_lengths, lengths, 256, cudaMemcpyHostToDevice, s), "lengths write");
    LWC_CUDA(cudaMemcpyAsync(blob + d.off_lut, plan.tables.data(), 2 * plan.tables.size(), cudaMemcpyHostToDevice, s),
             "lookup table write");
    // bytes no pass writes: unused chunk gaps, padding, the stream's tail (the
    // range after the gaps also clears the chunk counts, which lie between
    // the gaps and the block offsets and are accumulated by atomic adds)
    if (lwc_status st = zero(blob, d.off_lengths + 256, d.off_lut, s)) return st;
    if (lwc_status st = zero(blob, d.off_lut + 2 * plan.tables.size(), d.off_gaps, s)) return st;
    if (lwc_status st = zero(blob, d.off_gaps + d.n_chunks, d.off_blkoff, s)) return st;
    if (lwc_status st = zero(blob, d.off_blkoff + 8 * (d.n_blocks + 1), d.off_stream, s)) return st;
    if (lwc_status st = zero(blob, d.off_stream + 4 * stream_words, d.off_sm, s)) return st;

    WsHeader *ws = reinterpret_cast<WsHeader *>(work);
    uint32_t *tile_bits = reinterpret_cast<uint32_t *>(work + kWsArrays);
    uint64_t *tile_pos = reinterpret_cast<uint64_t *>(work + ws_tile_pos_off(n));
    uint32_t *stream = reinterpret_cast<uint32_t *>(blob + d.off_stream);
    unsigned grid;
    if (lwc_status st = grid_for((const void *)df11_tile_bits_kernel<E>, kTileThreads, 0, tiles, grid)) return st;
    df11_tile_bits_kernel<E><<<grid, kTileThreads, 0, s>>>(src, n, tiles, t, tile_bits, ws);
    LWC_CUDA(cudaGetLastError(), "encode launch");
    df11_scan_kernel<<<1, 1024, 0, s>>>(tile_bits, tile_pos, tiles, stream, stream_words, ws);
    LWC_CUDA(cudaGetLastError(), "encode launch");
    EmitArgs a;
    a.src = src;
    a.n = n;
    a.tile_pos = tile_pos;
    a.n_tiles = tiles;
    a.stream = stream;
    a.stream_words = stream_words;
    a.gaps = blob + d.off_gaps;
    a.counts = (d.flags & kFlagChunkCounts) ? reinterpret_cast<uint32_t *>(blob + d.off_counts) : nullptr;
    a.n_chunks = d.n_chunks;
    a.chunk_bits = 8ull * d.chunk_bytes;
    a.blkoff = reinterpret_cast<uint64_t *>(blob + d.off_blkoff);
    a.n_blocks = d.n_blocks;
    a.block_bits = a.chunk_bits * d.threads_per_block;
    a.sm = blob + d.off_sm;
    a.ws = ws;
    if (lwc_status st = grid_for((const void *)df11_emit_kernel<E>, kTileThreads, 0, tiles, grid)) return st;
    df11_emit_kernel<E><<<grid, kTileThreads, 0, s>>>(a, t);
    LWC_CUDA(cudaGetLastError(), "encode launch");
    const unsigned mgrid = (unsigned)std::min<uint64_t>(1024, (d.n_blocks + 255) / 256);
    df11_max_block_kernel<<<mgrid, 256, 0, s>>>(a.blkoff, d.n_blocks, ws);
    LWC_CUDA(cudaGetLastError(), "encode launch");

    WsHeader r;
    if (lwc_status st = fetch_header(work, r, nullptr, 0, s)) return st;
    if (r.error || r.total_bits != d.total_bits)
        return fail(LWC_ERR_INVALID_ARG, "source changed between plan and write (%llu bits planned, %llu found)",
                    (unsigned long long)d.total_bits, (unsigned long long)r.total_bits);
    d.max_block_count = r.max_block_count;
    return finish_blob(blob, d, desc_out, s);
}

lwc_status write_codebook(const uint16_t *src, uint64_t n, const WsHeader &h, const uint32_t *bitmap, uint8_t *work,
                          uint8_t *blob, uint64_t blob_bytes, lwc_desc *desc_out, cudaStream_t s) {
    uint32_t U = 0;
    for (uint32_t i = 0; i < 2048; i++) U += (uint32_t)__builtin_popcount(bitmap[i]);
    lwc_desc d;
    codebook_layout(U, n, d);
    if (blob_bytes < d.total_bytes)
        return fail(LWC_ERR_INVALID_ARG, "blob buffer of %llu bytes, %llu needed", (unsigned long long)blob_bytes,
                    (unsigned long long)d.total_bytes);
    WsHeader hw = h;
    hw.error = 0;
    if (lwc_status st = put_header(work, hw, s)) return st;
    WsHeader *ws = reinterpret_cast<WsHeader *>(work);
    uint16_t *rank = reinterpret_cast<uint16_t *>(work + kWsArrays);
    // table (into the blob) and index map (into the workspace) from the bitmap on the device
    cb_rank_kernel<<<kRankCtas, kRankThreads, 0, s>>>(reinterpret_cast<const uint32_t *>(work + kWsCounts), rank,
                                                      reinterpret_cast<uint16_t *>(blob + d.off_table), U, ws);
    LWC_CUDA(cudaGetLastError(), "encode launch");
    if (!d.k) {
        if (lwc_status st = zero(blob, d.off_table + 2ull * d.U, d.total_bytes, s)) return st;
    } else {
        const uint64_t packed_words = d.packed_bytes / 4, groups = (n + 1023) / 1024;
        const uint64_t written = std::min<uint64_t>(packed_words, groups * 32 * d.k);
        if (lwc_status st = zero(blob, d.off_table + 2ull * d.U, d.off_packed, s)) return st;
        if (lwc_status st = zero(blob, d.off_packed + 4 * written, d.total_bytes, s)) return st;
        const PackKernel kernel = kPackKernels[d.k - 1];
        unsigned grid;
        if (lwc_status st = grid_for((const void *)kernel, kPackWarps * 32, 0, (groups + kPackWarps - 1) / kPackWarps,
                                     grid))
            return st;
        kernel<<<grid, kPackWarps * 32, 0, s>>>(src, n, rank, d.U, reinterpret_cast<uint32_t *>(blob + d.off_packed),
                                               packed_words, ws);
        LWC_CUDA(cudaGetLastError(), "encode launch");
    }
    WsHeader r;
    if (lwc_status st = fetch_header(work, r, nullptr, 0, s)) return st;
    if (r.error) return fail(LWC_ERR_INVALID_ARG, "source changed between plan and write (unplanned 16-bit patterns)");
    return finish_blob(blob, d, desc_out, s);
}

}  // namespace
}  // namespace lwc

using namespace lwc;

extern "C" {

uint64_t lwc_encode_device_workspace_bytes(uint64_t n) { return workspace_bytes(n); }

lwc_status lwc_encode_dfloat11_elements_device_plan(const void *d_src, uint64_t n, uint32_t elem,
                                                    const lwc_df11_params *params, void *d_work, uint64_t work_bytes,
                                                    lwc_desc *desc_out, lwc_stream_t stream) {
    if (!desc_out) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    if (elem > LWC_ELEM_FP16) return fail(LWC_ERR_INVALID_ARG, "unknown element type %u", elem);
    if (lwc_status st = check_common(d_src, n, d_work, work_bytes)) return st;
    WsHeader h{};
    h.magic = kWsMagic;
    h.codec = LWC_CODEC_DFLOAT11;
    h.elem = elem;
    h.n = n;
    h.chunk_bytes = params ? params->chunk_bytes : kDefaultChunkBytes;
    h.threads_per_block = params ? params->threads_per_block : kDefaultThreadsPerBlock;
    h.max_len = params ? params->max_len : kDefaultMaxLen;
    h.chunk_counts = params ? (params->chunk_counts != 0) : kDefaultChunkCounts;
    if (lwc_status st = check_df11_params(h.chunk_bytes, h.threads_per_block, h.max_len)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *work = static_cast<uint8_t *>(d_work);
    LWC_CUDA(cudaMemsetAsync(work + kWsCounts, 0, 256 * sizeof(uint64_t), s), "memset");
    if (n) {
        const void *kernel = elem == LWC_ELEM_FP32   ? (const void *)df11_histogram_kernel<LWC_ELEM_FP32>
                             : elem == LWC_ELEM_FP16 ? (const void *)df11_histogram_kernel<LWC_ELEM_FP16>
                                                     : (const void *)df11_histogram_kernel<LWC_ELEM_BF16>;
        unsigned grid;
        if (lwc_status st = grid_for(kernel, 512, 0, (n / kPerThread + 511) / 512, grid)) return st;
        unsigned long long *counts = reinterpret_cast<unsigned long long *>(work + kWsCounts);
        if (elem == LWC_ELEM_FP32)
            df11_histogram_kernel<LWC_ELEM_FP32><<<grid, 512, 0, s>>>(d_src, n, counts);
        else if (elem == LWC_ELEM_FP16)
            df11_histogram_kernel<LWC_ELEM_FP16><<<grid, 512, 0, s>>>(d_src, n, counts);
        else
            df11_histogram_kernel<LWC_ELEM_BF16><<<grid, 512, 0, s>>>(d_src, n, counts);
        LWC_CUDA(cudaGetLastError(), "encode launch");
    }
    if (lwc_status st = put_header(work, h, s)) return st;
    uint64_t counts[256];
    WsHeader r;
    if (lwc_status st = fetch_header(work, r, counts, sizeof counts, s)) return st;
    Df11Plan plan;
    if (lwc_status st = plan_dfloat11(counts, n, h.chunk_bytes, h.threads_per_block, h.max_len, h.chunk_counts != 0,
                                      plan, lo_section_bytes(elem, n)))
        return st;
    plan.d.elem = elem;
    *desc_out = plan.d;
    clear_error();
    return LWC_OK;
}

lwc_status lwc_encode_dfloat11_device_plan(const void *d_src, uint64_t n, const lwc_df11_params *params,
                                           void *d_work, uint64_t work_bytes, lwc_desc *desc_out,
                                           lwc_stream_t stream) {
    return lwc_encode_dfloat11_elements_device_plan(d_src, n, LWC_ELEM_BF16, params, d_work, work_bytes, desc_out,
                                                    stream);
}

lwc_status lwc_encode_codebook_device_plan(const void *d_src, uint64_t n, void *d_work, uint64_t work_bytes,
                                           lwc_desc *desc_out, lwc_stream_t stream) {
    if (!desc_out) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    if (lwc_status st = check_common(d_src, n, d_work, work_bytes)) return st;
    WsHeader h{};
    h.magic = kWsMagic;
    h.codec = LWC_CODEC_CODEBOOK;
    h.n = n;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *work = static_cast<uint8_t *>(d_work);
    LWC_CUDA(cudaMemsetAsync(work + kWsCounts, 0, 8192, s), "memset");
    if (n) {
        unsigned grid;
        if (lwc_status st = grid_for((const void *)cb_presence_kernel, 512, 0, (n / 8 + 511) / 512, grid)) return st;
        cb_presence_kernel<<<grid, 512, 0, s>>>(static_cast<const uint16_t *>(d_src), n,
                                                reinterpret_cast<uint32_t *>(work + kWsCounts));
        LWC_CUDA(cudaGetLastError(), "encode launch");
    }
    if (lwc_status st = put_header(work, h, s)) return st;
    std::vector<uint32_t> bitmap(2048);
    WsHeader r;
    if (lwc_status st = fetch_header(work, r, bitmap.data(), 8192, s)) return st;
    uint32_t U = 0;
    for (uint32_t i = 0; i < 2048; i++) U += (uint32_t)__builtin_popcount(bitmap[i]);
    CbPlan plan;
    codebook_layout(U, n, plan.d);
    *desc_out = plan.d;
    clear_error();
    return LWC_OK;
}

lwc_status lwc_encode_device_write(const void *d_src, uint64_t n, void *d_work, uint64_t work_bytes, void *d_blob,
                                   uint64_t blob_bytes, lwc_desc *desc_out, lwc_stream_t stream) {
    if (!desc_out) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    if (lwc_status st = check_common(d_src, n, d_work, work_bytes)) return st;
    if (!d_blob) return fail(LWC_ERR_INVALID_ARG, "NULL blob buffer");
    if (!aligned16(d_blob)) return fail(LWC_ERR_MISALIGNED, "blob buffer must be 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *work = static_cast<uint8_t *>(d_work);
    std::vector<uint64_t> region(8192 / 8);
    WsHeader h;
    if (lwc_status st = fetch_header(work, h, region.data(), 8192, s)) return st;
    if (h.magic != kWsMagic || h.n != n)
        return fail(LWC_ERR_INVALID_ARG, "workspace holds no plan for this tensor (call a *_device_plan first)");
    lwc_status st;
    if (h.codec == LWC_CODEC_DFLOAT11 && h.elem == LWC_ELEM_FP32)
        st = write_dfloat11<LWC_ELEM_FP32>(d_src, n, h, region.data(), work, static_cast<uint8_t *>(d_blob), blob_bytes,
                                           desc_out, s);
    else if (h.codec == LWC_CODEC_DFLOAT11 && h.elem == LWC_ELEM_FP16)
        st = write_dfloat11<LWC_ELEM_FP16>(d_src, n, h, region.data(), work, static_cast<uint8_t *>(d_blob), blob_bytes,
                                           desc_out, s);
    else if (h.codec == LWC_CODEC_DFLOAT11 && h.elem == LWC_ELEM_BF16)
        st = write_dfloat11<LWC_ELEM_BF16>(d_src, n, h, region.data(), work, static_cast<uint8_t *>(d_blob), blob_bytes,
                                           desc_out, s);
    else if (h.codec == LWC_CODEC_CODEBOOK)
        st = write_codebook(static_cast<const uint16_t *>(d_src), n, h, reinterpret_cast<const uint32_t *>(region.data()),
                            work, static_cast<uint8_t *>(d_blob), blob_bytes, desc_out, s);
    else
        st = fail(LWC_ERR_INVALID_ARG, "workspace holds no plan (codec %u)", h.codec);
    if (st == LWC_OK) clear_error();
    return st;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation variant of the DFloat11 device encoder.
//
// For callers that cannot call cudaMalloc at encode time: typically a serving
// process whose memory manager has already reserved the device memory for
// weights and KV cache up front and allows no further cudaMalloc/cudaFree
// (a late cudaMalloc can fail or fragment the reserved pool, and cudaFree
// synchronises the whole device). Instead of a caller workspace this entry
// point uses one file-scope scratch array in device memory, created when the
// library's device code is loaded on a GPU and held by every GPU that loads
// it until the process exits.
namespace lwc {
namespace {

constexpr uint64_t kNoAllocMaxN = 1ull << 30;   // weights; every matrix of Llama-3-8B/70B fits
constexpr uint64_t kNoAllocScratchBytes = workspace_bytes(kNoAllocMaxN);
static_assert(kNoAllocScratchBytes == 3154432, "the scratch size stated in lwc.h");

// Shared by every call on a device; keeps the last call's contents (the plan
// step clears what must start at zero).
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices];

// Device address of the scratch array for the current device, looked up once
// per device (the symbol's host-side name is only a handle, not an address).
lwc_status noalloc_scratch(void *&ptr) {
    int dev = 0;
    LWC_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(LWC_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        LWC_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
        g_scratch_ptr[dev] = p;
    }
    ptr = g_scratch_ptr[dev];
    return LWC_OK;
}

}  // namespace
}  // namespace lwc

extern "C" lwc_status lwc_encode_dfloat11_device_noalloc(const void *d_src, uint64_t n, const lwc_df11_params *params,
                                                         void *d_blob, uint64_t blob_bytes, lwc_desc *desc_out,
                                                         lwc_stream_t stream) {
    if (!desc_out) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    if (n > kNoAllocMaxN)
        return fail(LWC_ERR_UNSUPPORTED,
                    "tensor of %llu weights is above the no-allocation encoder's maximum of %llu "
                    "(its scratch array holds %llu bytes)",
                    (unsigned long long)n, (unsigned long long)kNoAllocMaxN,
                    (unsigned long long)kNoAllocScratchBytes);
    if (!d_blob) return fail(LWC_ERR_INVALID_ARG, "NULL blob buffer");
    if (!aligned16(d_blob)) return fail(LWC_ERR_MISALIGNED, "blob buffer must be 16-byte aligned");
    void *scratch = nullptr;
    if (lwc_status st = noalloc_scratch(scratch)) return st;
    lwc_desc plan;
    if (lwc_status st = lwc_encode_dfloat11_device_plan(d_src, n, params, scratch, kNoAllocScratchBytes, &plan, stream))
        return st;
    if (blob_bytes < plan.total_bytes) {
        *desc_out = plan;   // tells the caller the size it needs
        return fail(LWC_ERR_INVALID_ARG, "blob buffer of %llu bytes, %llu needed", (unsigned long long)blob_bytes,
                    (unsigned long long)plan.total_bytes);
    }
    return lwc_encode_device_write(d_src, n, scratch, kNoAllocScratchBytes, d_blob, blob_bytes, desc_out, stream);
}
