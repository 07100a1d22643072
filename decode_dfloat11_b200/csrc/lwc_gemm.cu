// DFloat11 weights decoded straight into tensor-core operands: y = x W^T on
// the 5th-generation tensor cores (tcgen05) of sm_100a, for 1 to 256
// activation rows.
//
// What it computes: the linear layer that consumes the decompressed weights
// ("Koniec z kompromisami! DFloat11 ratuje dokładność modeli AI ...", section
// "Jak to działa w praktyce? Magia na poziomie GPU": the weights are
// decompressed on the GPU just before the layer uses them). The BF16 matrix
// never exists in HBM: each 128 x 64 tile of W is decoded into shared memory,
// in the layout the MMA reads, and consumed there.
//
// Weight order. The blob holds W (rows x cols, rows % 128 == 0, cols % 64 ==
// 0) in tile order: tile (i, j) = rows 128 i .. 128 i + 127, columns 64 j ..
// 64 j + 63, tiles ordered by i then j, each tile row-major (lwc_tile_order
// writes this order). The blob format itself is the plain DFloat11 one; so
// one work unit (128 rows of W, all columns) is a contiguous range of the
// decoded stream, whose k-tiles arrive in order.
//
// Roles (one CTA per SM, persistent; 5 + 4..20 warps, the host's choice by
// block size and shared memory):
//  * warps 5.. decode: they claim the unit's 32-chunk blocks in order (the
//    counted decoder: stored chunk counts, multi-code symbol tables), merge
//    each weight with its sign|mantissa byte and store it into the stage of
//    its k-tile, at its place in the 128-byte-swizzled K-major layout. The
//    warp that completes a tile signals it on the stage's barrier.
//  * warp 4, one thread, in an event loop: loads the x tile of each k-tile
//    with a tensor copy (no multicast), issues four tcgen05.mma per tile (M =
//    128 weight rows, N = the padded activation count, K = 16 each) with the
//    accumulator in tensor memory as soon as the tile is complete, and gives
//    each stage back to the decoders as soon as the MMAs that read it end.
//  * warps 0..3 (one per 32-lane quarter of tensor memory): after a unit's
//    last MMA, read its accumulator with tcgen05.ld and write y (FP32). Two
//    accumulators alternate, so this overlaps the next unit's MMAs.
// The units (128-row slices of every matrix of the call) are spread over the
// CTAs on the host, longest first onto the least loaded CTA, and passed in
// the launch parameters. Every wait is bounded; any failure raises a shared
// abort flag that ends every role's loop.
#include <cuda.h>   // CUtensorMap and its enums (the encode call is fetched at run time)
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "lwc_cb_dev.cuh"
#include "lwc_device.cuh"
#include "lwc_df11_dev.cuh"
#include "lwc_internal.h"
#include "lwc_umma.cuh"

namespace lwc {
namespace {

using namespace df11dev;
using namespace cbdev;

constexpr uint32_t kTileRows = 128;
constexpr uint32_t kTileCols = 64;
constexpr uint32_t kTileElems = kTileRows * kTileCols;   // 8192
constexpr uint32_t kTileBytes = kTileElems * 2;          // 16 KB
constexpr uint32_t kMaxMats = 8;           // matrices per call
constexpr uint32_t kMaxM = 256;            // activation rows (MMA N)
constexpr uint32_t kMaxUnits = 4096;       // 128-row units per call
constexpr uint32_t kMaxCtas = 256;
constexpr uint32_t kMaxCtaUnits = 64;      // units one CTA takes
constexpr uint32_t kMaxStages = 8;         // weight-tile stages
constexpr uint32_t kXStages = 2;           // x-tile stages (refilled from L2 by the tensor copy)
constexpr int kPreloadUnits = 8;           // 8-weight pieces per lane whose sign|mantissa loads are issued early
constexpr uint32_t kMaxDecWarps = 20;     // decoder warps: 25 warps leave 80 registers a thread (24 + 5 leave 64: spills)
constexpr uint32_t kInFlightWeights = 48 * 1024;   // blocks in flight: about six 8192-weight tiles
constexpr uint32_t kMinDecWarps = 4;
constexpr uint32_t kMaxCbK = 16;           // codebook index widths the product takes (1..16)
constexpr uint32_t kMmaWarp = 4;
constexpr uint32_t kDec0 = 5;              // first decoder warp
constexpr uint32_t kMaxCbDecWarps = 20;   // codebook decoder warps
constexpr uint32_t kMaxThreads = (kDec0 + kMaxDecWarps) * 32;
constexpr uint32_t kMaxCbThreads = (kDec0 + kMaxCbDecWarps) * 32;
constexpr uint32_t kDecBarrier = 1;        // named barrier of the decoder warps
// y of a matrix whose K range is split starts as this pattern (a NaN that no
// sum of finite or infinite products yields: those NaNs are canonical)
constexpr uint32_t kSplitEmpty = 0xFFFFFFFFu;

struct GemmMat {
    Df11Tensor t;          // DFloat11: the blob's sections (tile order); t.out unused
    const uint8_t *packed; // codebook: the k-bit indices (tile order)
    const uint16_t *table; // codebook: the table (U entries)
    uint32_t table_words;  // codebook: 32-bit words to copy from the table (2U bytes, rounded up)
    uint32_t pad;
    float *y;              // M x rows, row-major
    uint32_t rows, cols, k_tiles, kt_split;   // kt_split: k-tiles of part 0 when the K range is split, else 0
};

struct __align__(64) GemmBatch {
    CUtensorMap xmap[kMaxMats];   // x of each matrix: M x cols BF16, box 64 x n_pad, 128-byte swizzle
    GemmMat m[kMaxMats];
    uint32_t count, M, n_pad, stages;   // stages: weight-tile stages (x tiles have kXStages)
    uint32_t chunk_words, seg_words, stage_bytes, lut_entries;
    uint32_t tmem_cols, idesc, dec_warps, acc_cols;   // tensor memory: two accumulators of acc_cols columns
    uint32_t *status;
    uint16_t cta_begin[kMaxCtas + 1];   // CTA c takes sched[cta_begin[c] .. cta_begin[c + 1])
    uint16_t sched[kMaxUnits];          // matrix << 13 | part << 12 | 128-row unit index
};

__host__ __device__ constexpr uint32_t unit_mat(uint32_t u) { return u >> 13; }
__host__ __device__ constexpr uint32_t unit_part(uint32_t u) { return (u >> 12) & 1u; }
__host__ __device__ constexpr uint32_t unit_idx(uint32_t u) { return u & 0xFFFu; }

// The k-tiles a unit covers: all of them, or (split matrices) the first
// kt_split or the rest. In tile order a unit is one contiguous weight range.
struct UnitSpan {
    uint32_t mat, ru, part, kt0, kts;
    uint64_t lo;   // first weight of the unit (tile order)
};
__device__ __forceinline__ UnitSpan unit_span(const GemmBatch &B, uint32_t u) {
    UnitSpan r;
    r.mat = unit_mat(u);
    r.ru = unit_idx(u);
    r.part = unit_part(u);
    const GemmMat &g = B.m[r.mat];
    r.kt0 = r.part ? g.kt_split : 0u;
    r.kts = g.kt_split ? (r.part ? g.k_tiles - g.kt_split : g.kt_split) : g.k_tiles;
    r.lo = ((uint64_t)r.ru * g.k_tiles + r.kt0) * kTileElems;
    return r;
}

// Codebook decoder warps' shared memory: the table (2^k entries, so that
// every k-bit index stays inside it), two mbarriers and two task buffers per
// warp (a task = 1024 indices = 16 rows of a tile = 128 k bytes), a claim
// counter.
struct CbGemmLayout {
    uint32_t tab, bars, claim, bufs, total;
    __host__ __device__ CbGemmLayout(uint32_t k, uint32_t warps) {
        tab = 0;
        bars = (2u << k) < 16u ? 16u : (2u << k);
        claim = bars + ((16u * warps + 15u) & ~15u);
        bufs = claim + 16u;
        total = bufs + warps * 2u * 128u * k;
    }
};
__host__ __device__ inline uint32_t cb_dec_bytes(uint32_t k, uint32_t warps) { return CbGemmLayout(k, warps).total; }

// Shared memory of one CTA (offsets from a 1024-byte aligned base).
struct GemmLayout {
    uint32_t stage_stride, x_off, x_stride, dec, ctl, total;
    // control block (bytes from ctl)
    static constexpr uint32_t kFullX = 0;            // u64[kXStages]: x tile landed
    static constexpr uint32_t kFullW = 64;           // u64[kMaxStages]: weight tile complete
    static constexpr uint32_t kEmpty = 128;          // u64[kMaxStages]: the MMAs that read the stage completed
    static constexpr uint32_t kAccFull = 192;        // u64[2]: a unit's accumulator (buffer ui % 2) is final
    static constexpr uint32_t kAccEmpty = 208;       // u64[2]: the epilogue has read it
    static constexpr uint32_t kWritten = 224;        // u32[kMaxStages]: weights stored in the stage's tile
    static constexpr uint32_t kReleased = 256;       // u32[kMaxStages]: fills of the stage consumed
    static constexpr uint32_t kTmem = 288;           // u32: tensor-memory address
    static constexpr uint32_t kAbort = 292;          // u32
    static constexpr uint32_t kUnitFirst = 304;      // u32[kMaxCtaUnits]: a unit's first block
    static constexpr uint32_t kUnitItem = kUnitFirst + 4 * kMaxCtaUnits;   // u32[kMaxCtaUnits + 1]: first item
    static constexpr uint32_t kUnitTile = kUnitItem + 4 * (kMaxCtaUnits + 1) + 12;   // u32[kMaxCtaUnits + 1]
    static constexpr uint32_t kCtlBytes = kUnitTile + 4 * (kMaxCtaUnits + 1) + 12;
    // cb_k = 0: DFloat11 decoder warps (the counted decoder's layout); cb_k = k:
    // codebook decoder warps (CbGemmLayout)
    __host__ __device__ GemmLayout(uint32_t n_pad, uint32_t stages, uint32_t seg_words, uint32_t lut_entries,
                                   uint32_t stage_bytes, uint32_t dec_warps, uint32_t cb_k = 0) {
        stage_stride = kTileBytes;            // weight tiles, then x tiles; all multiples of 1024
        x_off = stages * stage_stride;
        x_stride = n_pad * 128u;
        dec = x_off + kXStages * x_stride;
        ctl = dec + (cb_k ? cb_dec_bytes(cb_k, dec_warps)
                          : CountedLayout(seg_words, lut_entries, stage_bytes, dec_warps).total);
        ctl = (ctl + 15u) & ~15u;
        total = ctl + kCtlBytes;
    }
};

__device__ __forceinline__ void dec_sync(uint32_t threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(kDecBarrier), "r"(threads) : "memory");
}

// Bounded wait on an mbarrier phase that also gives up when the CTA aborts.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, const volatile uint32_t *abort) {
    for (uint32_t i = 0; i < dev::kWaitPolls; ++i) {
        if (dev::mbar_try_wait(bar, parity)) return true;
        if ((i & 15u) == 15u && *abort) return false;
    }
    return false;
}

// Bounded wait until a counter in shared memory reaches `need`.
__device__ __forceinline__ bool wait_count(const volatile uint32_t *c, uint32_t need, const volatile uint32_t *abort) {
    for (uint32_t i = 0; i < dev::kWaitPolls; ++i) {
        if (*c >= need) return true;
        if (*abort) return false;
        __nanosleep(64);
    }
    return false;
}

// The abort flag as lane 0 reads it, so that the whole warp takes one path.
__device__ __forceinline__ bool warp_aborted(const volatile uint32_t *abort) {
    return __shfl_sync(0xFFFFFFFFu, *abort, 0) != 0;
}

__device__ __forceinline__ void st_shared_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"((unsigned short)v) : "memory");
}

// One BF16 weight from its sign|mantissa byte s and its rotated exponent r
// (r = e >> 1 | (e & 1) << 7): low byte = s's mantissa under r's top bit,
// high byte = r's low seven bits under s's sign bit.
__device__ __forceinline__ uint32_t merge1r(uint32_t s, uint32_t r) {
    return ((s & 0x7Fu) | (r & 0x80u)) | (((r & 0x7Fu) | (s & 0x80u)) << 8);
}

// The kernel body; CBK = 0: DFloat11 weights, CBK = k: codebook weights with
// k-bit indices (only the decoder warps differ).
template <int CBK>
__device__ __forceinline__ void gemm_body(const GemmBatch &B) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const uint32_t raw_a = dev::smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_a + 1023u) & ~1023u) - raw_a);   // tiles need 1024-byte alignment
    const uint32_t NS = B.stages;
    const GemmLayout G(B.n_pad, NS, B.seg_words, B.lut_entries, B.stage_bytes, B.dec_warps, CBK);
    uint8_t *ctl = smem + G.ctl;
    uint64_t *full_x = reinterpret_cast<uint64_t *>(ctl + GemmLayout::kFullX);
    uint64_t *full_w = reinterpret_cast<uint64_t *>(ctl + GemmLayout::kFullW);
    uint64_t *empty = reinterpret_cast<uint64_t *>(ctl + GemmLayout::kEmpty);
    uint64_t *acc_full = reinterpret_cast<uint64_t *>(ctl + GemmLayout::kAccFull);
    uint64_t *acc_empty = reinterpret_cast<uint64_t *>(ctl + GemmLayout::kAccEmpty);
    uint32_t *written = reinterpret_cast<uint32_t *>(ctl + GemmLayout::kWritten);
    volatile uint32_t *released = reinterpret_cast<volatile uint32_t *>(ctl + GemmLayout::kReleased);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(ctl + GemmLayout::kTmem);
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(ctl + GemmLayout::kAbort);
    uint32_t *u_first = reinterpret_cast<uint32_t *>(ctl + GemmLayout::kUnitFirst);
    uint32_t *u_item = reinterpret_cast<uint32_t *>(ctl + GemmLayout::kUnitItem);
    uint32_t *u_tile = reinterpret_cast<uint32_t *>(ctl + GemmLayout::kUnitTile);

    const uint32_t c0 = B.cta_begin[blockIdx.x];
    const uint32_t nunits = B.cta_begin[blockIdx.x + 1] - c0;
    uint32_t bad = 0;

    // ---- prologue: barriers, counters, tensor memory, this CTA's unit table
    if (tid == 0) {
        for (uint32_t s = 0; s < kXStages; s++) dev::mbar_init(&full_x[s], 1);
        for (uint32_t s = 0; s < NS; s++) {
            dev::mbar_init(&full_w[s], 1);
            dev::mbar_init(&empty[s], 1);
            written[s] = 0;
            released[s] = 0;
        }
        for (uint32_t k = 0; k < 2; k++) {
            dev::mbar_init(&acc_full[k], 1);
            dev::mbar_init(&acc_empty[k], 4);
        }
        *abort_flag = 0;
        dev::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        umma::tmem_alloc(tmem_slot, B.tmem_cols);
        umma::tmem_relinquish();
    }
    for (uint32_t i = tid; i < nunits; i += blockDim.x) {
        const UnitSpan sp = unit_span(B, B.sched[c0 + i]);
        u_tile[i + 1] = sp.kts;
        if constexpr (CBK != 0) {   // codebook decoders take whole tiles: no blocks to find
            u_first[i] = 0;
            u_item[i + 1] = 0;
            continue;
        }
        const GemmMat &gm = B.m[sp.mat];
        const uint64_t lo = sp.lo, hi = lo + (uint64_t)sp.kts * kTileElems;
        // the last block whose first weight is <= v (block 0 starts at weight 0)
        auto last_le = [&](uint64_t v) {
            uint32_t a = 0, b = gm.t.n_blocks;
            while (b - a > 1) {
                const uint32_t mid = a + (b - a) / 2;
                if (gm.t.blkoff[mid] <= v) a = mid; else b = mid;
            }
            return a;
        };
        const uint32_t first = last_le(lo), last = last_le(hi - 1);
        // block offsets that are not ascending (a damaged blob) can give last < first:
        // the unit gets no items and is reported below
        u_first[i] = last >= first ? first : 0xFFFFFFFFu;
        u_item[i + 1] = last >= first ? last - first + 1 : 0u;
    }
    __syncthreads();
    if (tid == 0) {
        u_item[0] = 0;
        u_tile[0] = 0;
        for (uint32_t i = 0; i < nunits; i++) {
            if (u_first[i] == 0xFFFFFFFFu) {
                bad |= LWC_DEVICE_BAD_OFFSET;
                *abort_flag = 1;
                u_first[i] = 0;
            }
            u_item[i + 1] += u_item[i];
            u_tile[i + 1] += u_tile[i];
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tiles_a = dev::smem_u32(smem);   // weight tile of stage s at tiles_a + s * stride
    const uint32_t tiles_x = tiles_a + G.x_off;      // x tile of x stage k at tiles_x + k * x_stride

    if (warp == kMmaWarp) {
        // ---- one thread: x tiles by tensor copy, MMAs, stage release
        if (lane == 0) {
            const uint32_t T = u_tile[nunits];
            const uint32_t xbytes = B.n_pad * 128u;
            uint32_t lq = 0, lu = 0, lk = 0;   // next tile whose x tile is loaded: its unit and k-tile
            auto load_x = [&]() {
                const uint32_t s = lq % kXStages;
                const UnitSpan sp = unit_span(B, B.sched[c0 + lu]);
                dev::mbar_arrive_expect_tx(&full_x[s], xbytes);
                umma::tma_load_2d(smem + G.x_off + s * G.x_stride, &B.xmap[sp.mat],
                                  (int32_t)((sp.kt0 + lk) * kTileCols), 0, &full_x[s]);
                lq++;
                if (++lk == sp.kts) {
                    lk = 0;
                    lu++;
                }
            };
            for (uint32_t j = 0; j < kXStages && lq < T; j++) load_x();
            // Event loop: retire the oldest issued tile as soon as its MMAs complete
            // (its weight stage goes back to the decoders, its x stage takes the tile
            // kXStages ahead), and issue the next tile as soon as its weights and x are in.
            // Phase parities are unambiguous: a stage's barriers never run more than
            // one fill ahead of this thread.
            uint32_t issued = 0, retired = 0, ui = 0, kt = 0, idle = 0;
            uint32_t KT = nunits ? unit_span(B, B.sched[c0]).kts : 0u;
            bool ok = true;
            while (retired < T) {
                bool progress = false;
                if (retired < issued && dev::mbar_test(&empty[retired % NS], (retired / NS) & 1u)) {
                    __threadfence_block();
                    released[retired % NS] = retired / NS + 1;
                    retired++;
                    if (lq < T) load_x();
                    progress = true;
                }
                if (issued < T && issued - retired < NS) {
                    const uint32_t s = issued % NS, f = issued / NS, sx = issued % kXStages;
                    // unit ui accumulates in buffer ui % 2, free once the epilogue has read unit ui - 2
                    if (dev::mbar_test(&full_x[sx], (issued / kXStages) & 1u) && dev::mbar_test(&full_w[s], f & 1u) &&
                        (kt != 0 || ui < 2 || dev::mbar_test(&acc_empty[ui & 1u], ((ui >> 1) - 1) & 1u))) {
                        umma::fence_after_sync();
                        const uint32_t a = tiles_a + s * G.stage_stride, b = tiles_x + sx * G.x_stride;
                        const uint32_t d = tmem + (ui & 1u) * B.acc_cols;
#pragma unroll
                        for (uint32_t k = 0; k < kTileCols / 16; k++)
                            umma::mma_bf16(d, umma::smem_desc_sw128(a + 32u * k), umma::smem_desc_sw128(b + 32u * k),
                                           B.idesc, (kt | k) != 0);
                        umma::mma_commit(&empty[s]);
                        if (kt + 1 == KT) umma::mma_commit(&acc_full[ui & 1u]);   // the unit's accumulator, once complete
                        issued++;
                        if (++kt == KT) {
                            kt = 0;
                            ui++;
                            KT = ui < nunits ? unit_span(B, B.sched[c0 + ui]).kts : 0u;
                        }
                        progress = true;
                    }
                }
                if (progress) {
                    idle = 0;
                } else {
                    if (++idle >= dev::kWaitPolls || ((idle & 63u) == 0 && *abort_flag)) {
                        ok = false;
                        break;
                    }
                    __nanosleep(32);
                }
            }
            if (!ok) {
                if (!*abort_flag) bad |= LWC_DEVICE_TIMEOUT;
                *abort_flag = 1;
            }
            // before the CTA ends: every issued MMA completes, every x tile in flight lands
            while (retired < issued && dev::mbar_wait_bounded(&empty[retired % NS], (retired / NS) & 1u)) retired++;
            for (uint32_t r = issued; r < lq; r++) dev::mbar_wait_bounded(&full_x[r % kXStages], (r / kXStages) & 1u);
        }
        __syncwarp();
    } else if (warp < kMmaWarp) {
        // ---- epilogue: warp w reads accumulator lanes 32 w .. 32 w + 31 (weight rows)
        for (uint32_t ui = 0; ui < nunits; ui++) {
            if (!wait_phase(&acc_full[ui & 1u], (ui >> 1) & 1u, abort_flag)) {
                if (!*abort_flag) bad |= LWC_DEVICE_TIMEOUT;
                *abort_flag = 1;
                break;
            }
            umma::fence_after_sync();
            const uint32_t u = B.sched[c0 + ui];
            const GemmMat &gm = B.m[unit_mat(u)];
            float *y = gm.y + (unit_idx(u) * kTileRows + warp * 32u + lane);
            const uint32_t taddr = tmem + ((warp * 32u) << 16) + (ui & 1u) * B.acc_cols;
            const bool split = gm.kt_split != 0;
            for (uint32_t c = 0; c < B.n_pad; c += 16) {
                uint32_t v[16];
                umma::tmem_ld16(taddr + c, v);
#pragma unroll
                for (uint32_t j = 0; j < 16; j++) {
                    if (c + j >= B.M) continue;
                    float *py = y + (size_t)(c + j) * gm.rows;
                    if (!split) {
                        *py = __uint_as_float(v[j]);
                    } else {
                        // the K range is split in two parts: y starts as kSplitEmpty; the part
                        // that finds the other's product there stores the sum (IEEE addition
                        // commutes, so the result does not depend on which part came second)
                        const uint32_t other = atomicExch(reinterpret_cast<unsigned int *>(py), v[j]);
                        if (other != kSplitEmpty) *py = __uint_as_float(v[j]) + __uint_as_float(other);
                    }
                }
            }
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0) dev::mbar_arrive(&acc_empty[ui & 1u]);
        }
    } else if constexpr (CBK == 0) {
        // ---- decoder warps: blocks of this CTA's units, in order, into the stages
        const uint32_t dw = warp - kDec0, dt = tid - kDec0 * 32u;
        const uint32_t DW = B.dec_warps, DT = DW * 32u;
        const CountedLayout L(B.seg_words, B.lut_entries, B.stage_bytes, DW);
        uint8_t *dsm = smem + G.dec;
        uint2 *sym = reinterpret_cast<uint2 *>(dsm);
        uint32_t *sub = reinterpret_cast<uint32_t *>(dsm + kFastSize * 8);
        uint16_t *lut = reinterpret_cast<uint16_t *>(dsm + kCtdTabBytes);
        uint8_t *buf = dsm + L.warp0 + dw * L.warp_bytes;
        const uint32_t *seg = reinterpret_cast<const uint32_t *>(buf);
        const uint8_t *gapb = buf + L.gaps;
        const uint8_t *cntb = buf + L.counts;
        uint32_t *slot = reinterpret_cast<uint32_t *>(buf + L.slot) + lane;
        const uint32_t slot_a = dev::smem_u32(slot), stage_a = dev::smem_u32(buf + L.stage);
        const uint8_t *stage = buf + L.stage;
        uint32_t *first_long = reinterpret_cast<uint32_t *>(dsm + L.misc);
        uint32_t *claim = first_long + 1;   // the next unclaimed item of the current matrix
        uint64_t *bar = reinterpret_cast<uint64_t *>(dsm + L.bars) + dw;
        const uint32_t seg_bytes = L.seg_bytes, last = B.seg_words - 1, cbits = B.chunk_words * 32u;
        if (lane == 0) {
            dev::mbar_init(bar, 1);
            dev::fence_mbar_init();
        }
        __syncwarp();
        uint32_t items = 0;   // copies issued on this warp's barrier (one phase each)
        // Every decoder warp walks every run of units that share a matrix and
        // passes the same named barriers, aborting or not.
        for (uint32_t i0 = 0; i0 < nunits;) {
            const uint32_t mat = unit_mat(B.sched[c0 + i0]);
            uint32_t i1 = i0 + 1;
            while (i1 < nunits && unit_mat(B.sched[c0 + i1]) == mat) i1++;
            const GemmMat &gm = B.m[mat];
            const Df11Tensor &tn = gm.t;
            const uint32_t ib = u_item[i0], ie = u_item[i1];
            // the unit of an item of this run, searching forward from unit `from`
            auto unit_of = [&](uint32_t item, uint32_t from) {
                while (from + 1 < i1 && u_item[from + 1] <= item) from++;
                return from;
            };
            dec_sync(DT);   // every decoder warp is done with the previous tables and its own buffers
            if (dt == 0) *claim = ib + DW;
            // warps take the run's first items in order, then claim one at a time;
            // the first item's copies overlap the table build
            uint32_t w = ib + dw, ui = i0, bn = 0;
            uint64_t o0n = 0, o1n = 0;
            if (w < ie && !warp_aborted(abort_flag)) {
                ui = unit_of(w, ui);
                bn = u_first[ui] + (w - u_item[ui]);
                o0n = tn.blkoff[bn];
                o1n = tn.blkoff[bn + 1];
                issue_counted_item(tn, B.chunk_words, bn, buf, seg_bytes, bar, lane);
            } else {
                w = ie;
            }
            const uint32_t ntab = min(tn.n_tables, B.lut_entries / 256u);
            for (uint32_t i = dt; i < ntab * 128u; i += DT)
                reinterpret_cast<uint32_t *>(lut)[i] = reinterpret_cast<const uint32_t *>(tn.lut)[i];
            dec_sync(DT);
            build_counted_tables(lut, ntab, sym, sub, first_long, dt, DT, [DT] { dec_sync(DT); });
            dec_sync(DT);
            const uint32_t v0 = *first_long;

            // invariant at the loop top: the copies of item w (w < ie) are in flight
            while (w < ie && !warp_aborted(abort_flag)) {
                const uint32_t b = bn, cu = ui;
                const uint64_t o0 = o0n, o1 = o1n;
                uint32_t wn = 0;
                if (lane == 0) wn = atomicAdd(claim, 1u);
                wn = __shfl_sync(0xFFFFFFFFu, wn, 0);
                const bool more = wn < ie;
                if (more) {
                    ui = unit_of(wn, ui);
                    bn = u_first[ui] + (wn - u_item[ui]);
                    o0n = tn.blkoff[bn];
                    o1n = tn.blkoff[bn + 1];
                }
                const UnitSpan usp = unit_span(B, B.sched[c0 + cu]);
                const uint64_t ulo = usp.lo, uhi = ulo + (uint64_t)usp.kts * kTileElems;
                const bool ok = o0 <= o1 && o1 <= tn.n && o1 - o0 + 16 <= B.stage_bytes && o0 < uhi && o1 > ulo;
                const uint64_t p_lo = ok ? max(o0, ulo) : 0, p_hi = ok ? min(o1, uhi) : 0;
                // this unit's part of the block: 8-weight pieces [g_lo, g_hi), single weights at either end
                const uint64_t g_lo = (p_lo + 7) & ~7ull, g_hi = p_hi & ~7ull;
                const uint32_t nu = g_hi > g_lo ? (uint32_t)((g_hi - g_lo) >> 3) : 0u;
                const uint64_t i1 = lane < 8 ? p_lo + lane : max(g_hi, g_lo) + (lane - 8);
                const bool one = ok && (lane < 8 ? i1 < min(g_lo, p_hi) : (lane < 16 && i1 < p_hi));
                // the sign|mantissa bytes of this lane's first pieces are loaded now, under the copy and the decode
                uint2 sv[kPreloadUnits];
#pragma unroll
                for (int m = 0; m < kPreloadUnits; m++) {
                    const uint32_t j = lane + 32u * (uint32_t)m;
                    sv[m] = j < nu ? __ldg(reinterpret_cast<const uint2 *>(tn.sm + g_lo + 8ull * j)) : make_uint2(0, 0);
                }
                const uint32_t s1 = one ? tn.sm[i1] : 0u;
                if (lane == 0 && nu > 32u * kPreloadUnits && p_hi - p_lo < (1u << 20))   // the rest into L2
                    dev::prefetch_l2(tn.sm + (p_lo & ~15ull), (uint32_t)(((p_hi + 15) & ~15ull) - (p_lo & ~15ull)));
                const bool arrived = dev::mbar_wait_bounded(bar, items & 1u);
                items++;
                if (__any_sync(0xFFFFFFFFu, !arrived)) {
                    // let the late copy land (bounded) before this warp stops
                    bad |= LWC_DEVICE_TIMEOUT;
                    if (lane == 0) dev::mbar_wait_bounded(bar, (items - 1) & 1u);
                    *abort_flag = 1;
                    w = ie;
                    break;
                }
                bool next_issued = false, good = false;
                if (!ok) {
                    bad |= LWC_DEVICE_BAD_OFFSET;
                } else {
                    // output positions: a warp scan of the stored counts
                    const uint32_t cnt = cntb[lane];
                    uint32_t x = cnt;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
                        if (lane >= (uint32_t)o) x += y;
                    }
                    const uint32_t total = __shfl_sync(0xFFFFFFFFu, x, 31);
                    if (total != (uint32_t)(o1 - o0)) {
                        bad |= LWC_DEVICE_BAD_COUNT;
                    } else {
                        const uint32_t first = x - cnt;
                        const uint32_t qb = (uint32_t)(o0 & 15u) + first;   // staging byte of this lane's first exponent
                        const uint64_t rem_block = tn.total_bits - (uint64_t)b * 32u * cbits;
                        const uint32_t start = lane * cbits + gapb[lane];
                        const bool has_next = lane + 1 < 32u || b + 1 < tn.n_blocks;
                        const uint64_t next = has_next ? (uint64_t)(lane + 1) * cbits + gapb[lane + 1] : rem_block;
                        const uint32_t end = (uint32_t)min(next, rem_block);
                        uint32_t bad_here = 0;
                        if (cnt) {
                            const uint32_t got = decode_counted(seg, last, sym, sub, v0, lut, ntab, start, cnt, qb,
                                                                stage_a, slot_a, bad_here);
                            if (got - end > 40u) bad_here |= LWC_DEVICE_BAD_COUNT;
                        }
                        __syncwarp();
                        if ((qb & 3u) && cnt) {   // the bytes of this lane's first, shared word
                            const uint32_t hw = *slot, j0 = qb & 3u;
                            uint8_t *hb = buf + L.stage + (qb & ~3u);
                            hb[j0] = (uint8_t)(hw >> (8 * j0));
                            if (j0 < 3 && cnt > 1) hb[j0 + 1] = (uint8_t)(hw >> (8 * j0 + 8));
                            if (j0 == 1 && cnt > 2) hb[3] = (uint8_t)(hw >> 24);
                        }
                        __syncwarp();
                        // the segment is free: fetch this warp's next block while merging this one
                        if (more) issue_counted_item(tn, B.chunk_words, bn, buf, seg_bytes, bar, lane);
                        next_issued = true;
                        bad |= bad_here;
                        const bool clean = !__any_sync(0xFFFFFFFFu, bad_here != 0);
                        // the tiles (tile sequence numbers) this block writes, and their stages' turn
                        const uint32_t t0 = u_tile[cu];
                        const uint32_t qa = t0 + (uint32_t)((p_lo - ulo) / kTileElems);
                        const uint32_t qz = t0 + (uint32_t)((p_hi - 1 - ulo) / kTileElems);
                        uint32_t free_ = 0;
                        if (lane == 0 && clean)
                            free_ = wait_count(&released[qa % NS], qa / NS, abort_flag) &&
                                    (qz == qa || wait_count(&released[qz % NS], qz / NS, abort_flag));
                        free_ = __shfl_sync(0xFFFFFFFFu, free_, 0);
                        if (free_) {
                            __threadfence_block();
                            const uint64_t base = o0 & ~15ull;
                            // the stages of the block's first and (if it has one) second tile; t = weight
                            // index in the unit, tiles start every kTileElems
                            const uint32_t st_a = tiles_a + (qa % NS) * G.stage_stride;
                            const uint32_t st_z = tiles_a + (qz % NS) * G.stage_stride;
                            const uint32_t t_split = (qa + 1 - t0) * kTileElems;
                            const uint32_t tg = (uint32_t)(g_lo - ulo), eg = (uint32_t)(g_lo - base);
                            // 8-weight piece j: one 16-byte chunk of a swizzled tile row
                            auto put8 = [&](uint32_t j, uint2 sm8) {
                                const uint32_t t = tg + 8u * j;
                                const uint2 ev = *reinterpret_cast<const uint2 *>(stage + eg + 8u * j);
                                uint32_t w0, w1, w2, w3;
                                merge4r(sm8.x, ev.x, w0, w1);
                                merge4r(sm8.y, ev.y, w2, w3);
                                const uint32_t idx = t & (kTileElems - 1u);
                                st_shared_v4((t < t_split ? st_a : st_z) + umma::sw128_offset(idx >> 6, idx & 63u), w0, w1,
                                             w2, w3);
                            };
#pragma unroll
                            for (int m = 0; m < kPreloadUnits; m++) {
                                const uint32_t j = lane + 32u * (uint32_t)m;
                                if (j < nu) put8(j, sv[m]);
                            }
                            // the rest (blocks of more than 2048 weights), loads issued four at a time
                            for (uint32_t j0 = lane + 32u * kPreloadUnits; j0 < nu; j0 += 128u) {
                                uint2 r4[4];
#pragma unroll
                                for (uint32_t k = 0; k < 4; k++) {
                                    const uint32_t j = j0 + 32u * k;
                                    r4[k] = j < nu ? __ldg(reinterpret_cast<const uint2 *>(tn.sm + g_lo + 8ull * j))
                                                   : make_uint2(0, 0);
                                }
#pragma unroll
                                for (uint32_t k = 0; k < 4; k++)
                                    if (j0 + 32u * k < nu) put8(j0 + 32u * k, r4[k]);
                            }
                            // single weights before the first piece (lanes 0-7) and after the last (lanes 8-15)
                            if (one) {
                                const uint32_t t = (uint32_t)(i1 - ulo), idx = t & (kTileElems - 1u);
                                st_shared_u16((t < t_split ? st_a : st_z) + umma::sw128_offset(idx >> 6, idx & 63u),
                                              merge1r(s1, stage[i1 - base]));
                            }
                            dev::fence_proxy_async_smem();   // these stores before the MMA's (async-proxy) reads
                            __syncwarp();
                            if (lane == 0) {
                                __threadfence_block();
                                for (uint32_t q = qa; q <= qz; q++) {
                                    const uint64_t tlo = ulo + (uint64_t)(q - t0) * kTileElems;
                                    const uint32_t n_in = (uint32_t)(min(p_hi, tlo + kTileElems) - max(p_lo, tlo));
                                    const uint32_t s = q % NS;
                                    const uint32_t now = atomicAdd(&written[s], n_in) + n_in;
                                    if (now == kTileElems) {   // the tile is complete
                                        written[s] = 0;
                                        __threadfence_block();
                                        dev::mbar_arrive(&full_w[s]);
                                    } else if (now > kTileElems) {   // blocks overlap: a damaged blob
                                        bad |= LWC_DEVICE_BAD_OFFSET;
                                        *abort_flag = 1;
                                    }
                                }
                            }
                            good = true;
                        }
                    }
                }
                __syncwarp();
                if (!good) {
                    *abort_flag = 1;
                    w = next_issued && more ? wn : ie;   // a copy still in flight is waited for below
                    break;
                }
                w = more ? wn : ie;
            }
            if (w < ie) {   // the copies of item w were issued: let them land (bounded)
                if (lane == 0) dev::mbar_wait_bounded(bar, items & 1u);
                items++;
                __syncwarp();
            }
            i0 = i1;
        }
    } else {
        // ---- codebook decoder warps: tasks of 1024 indices (16 rows of a tile), in
        // tile order, each bulk-copied into one of the warp's two buffers, unpacked
        // (32 fields of k bits per lane), gathered from the table and stored as four
        // 16-byte chunks at their swizzled places in the tile's stage
        constexpr uint32_t K = CBK, kTaskBytes = 128u * K, kTaskWords = 32u * K;
        const uint32_t DW = B.dec_warps, DT = DW * 32u, dw = warp - kDec0, dt = tid - kDec0 * 32u;
        const CbGemmLayout C(K, DW);
        uint8_t *dsm = smem + G.dec;
        uint16_t *tab = reinterpret_cast<uint16_t *>(dsm + C.tab);
        uint64_t *cbar = reinterpret_cast<uint64_t *>(dsm + C.bars) + 2 * dw;
        uint32_t *claim = reinterpret_cast<uint32_t *>(dsm + C.claim);
        uint32_t *bufs = reinterpret_cast<uint32_t *>(dsm + C.bufs) + dw * 2u * kTaskWords;
        if (lane == 0) {
            dev::mbar_init(&cbar[0], 1);
            dev::mbar_init(&cbar[1], 1);
            dev::fence_mbar_init();
        }
        __syncwarp();
        uint32_t copies = 0;   // copies issued; copy c uses buffer and barrier c % 2, phase (c / 2) & 1
        // lane 0: the bulk copy of task t's packed indices into buffer `copies % 2`
        auto issue = [&](uint32_t t, uint32_t ui) {
            if (lane == 0) {
                const UnitSpan sp = unit_span(B, B.sched[c0 + ui]);
                const GemmMat &g = B.m[sp.mat];
                const uint64_t tile = (uint64_t)sp.ru * g.k_tiles + sp.kt0 + (t / 8u - u_tile[ui]);
                const uint32_t b = copies & 1u;
                dev::fence_proxy_async_smem();   // this warp's reads of the buffer come before the copy's writes
                dev::mbar_arrive_expect_tx(&cbar[b], kTaskBytes);
                dev::bulk_g2s(bufs + b * kTaskWords, g.packed + tile * (8u * kTaskBytes) + (t % 8u) * kTaskBytes,
                              kTaskBytes, &cbar[b]);
            }
            copies++;
        };
        for (uint32_t i0 = 0; i0 < nunits;) {
            const uint32_t mat = unit_mat(B.sched[c0 + i0]);
            uint32_t i1 = i0 + 1;
            while (i1 < nunits && unit_mat(B.sched[c0 + i1]) == mat) i1++;
            const GemmMat &gm = B.m[mat];
            const uint32_t tb = 8u * u_tile[i0], te = 8u * u_tile[i1];   // this run's tasks
            auto unit_of = [&](uint32_t t, uint32_t from) {
                while (from + 1 < i1 && 8u * u_tile[from + 1] <= t) from++;
                return from;
            };
            dec_sync(DT);   // every decoder warp is done with the previous table
            for (uint32_t i = dt; i < gm.table_words; i += DT)
                reinterpret_cast<uint32_t *>(tab)[i] = reinterpret_cast<const uint32_t *>(gm.table)[i];
            if (dt == 0) *claim = tb + DW;
            dec_sync(DT);
            uint32_t t = tb + dw, ui = i0;
            if (t < te && !warp_aborted(abort_flag)) {
                ui = unit_of(t, ui);
                issue(t, ui);
            } else {
                t = te;
            }
            // invariant at the loop top: the copy of task t (t < te) is copy `copies - 1`
            while (t < te && !warp_aborted(abort_flag)) {
                const uint32_t cur = copies - 1u;
                uint32_t tn = 0;
                if (lane == 0) tn = atomicAdd(claim, 1u);
                tn = __shfl_sync(0xFFFFFFFFu, tn, 0);
                if (tn < te) {   // the next task's copy, into the other buffer
                    ui = unit_of(tn, ui);
                    issue(tn, ui);
                }
                const uint32_t q = t / 8u, s = q % NS;
                uint32_t free_ = 0;
                if (lane == 0) free_ = wait_count(&released[s], q / NS, abort_flag);
                free_ = __shfl_sync(0xFFFFFFFFu, free_, 0);
                const bool landed = dev::mbar_wait_bounded(&cbar[cur & 1u], (cur >> 1) & 1u);
                if (__any_sync(0xFFFFFFFFu, !landed)) {
                    bad |= LWC_DEVICE_TIMEOUT;
                    if (lane == 0) dev::mbar_wait_bounded(&cbar[cur & 1u], (cur >> 1) & 1u);
                }
                if (!free_ || __any_sync(0xFFFFFFFFu, !landed)) {
                    *abort_flag = 1;
                    t = tn < te ? tn : te;   // a copy still in flight is waited for below
                    break;
                }
                uint32_t wv[K + 1];
                load_words<K>(bufs + (cur & 1u) * kTaskWords + lane * K, wv);
                uint32_t o[16];
                Gather<K, 0>::run(wv, tab, o);
                __syncwarp();   // the buffer is free for the copy after next
                // 32 weights: row 16 (t % 8) + lane / 2 of the tile, columns 32 (lane % 2) .. + 31
                const uint32_t r = 16u * (t % 8u) + (lane >> 1), c8 = (lane & 1u) * 4u;
                const uint32_t row = tiles_a + s * G.stage_stride + r * 128u;
#pragma unroll
                for (uint32_t k = 0; k < 4; k++)
                    st_shared_v4(row + ((((c8 + k) ^ r) & 7u) << 4), o[4 * k], o[4 * k + 1], o[4 * k + 2],
                                 o[4 * k + 3]);
                dev::fence_proxy_async_smem();   // these stores before the MMA's (async-proxy) reads
                __syncwarp();
                if (lane == 0) {
                    __threadfence_block();
                    const uint32_t now = atomicAdd(&written[s], 1024u) + 1024u;
                    if (now == kTileElems) {   // the tile is complete
                        written[s] = 0;
                        __threadfence_block();
                        dev::mbar_arrive(&full_w[s]);
                    }
                }
                t = tn < te ? tn : te;
            }
            if (t < te) {   // the copy of task t was issued: let it land (bounded)
                if (lane == 0) dev::mbar_wait_bounded(&cbar[(copies - 1u) & 1u], ((copies - 1u) >> 1) & 1u);
                __syncwarp();
            }
            i0 = i1;
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, B.tmem_cols);
    }
    if (bad && B.status) atomicOr(B.status, bad);
}

__global__ void __launch_bounds__(kMaxThreads, 1) df11_gemm_kernel(const __grid_constant__ GemmBatch B) {
    gemm_body<0>(B);
}

template <int K>
__global__ void __launch_bounds__(kMaxCbThreads, 1) cb_gemm_kernel(const __grid_constant__ GemmBatch B) {
    gemm_body<K>(B);
}

template <int K>
void launch_cb_gemm(const GemmBatch &B, dim3 grid, dim3 block, size_t smem, cudaStream_t s) {
    cb_gemm_kernel<K><<<grid, block, smem, s>>>(B);
}
using CbGemmLaunch = void (*)(const GemmBatch &, dim3, dim3, size_t, cudaStream_t);
const CbGemmLaunch kCbGemmKernels[kMaxCbK + 1] = {
    nullptr, launch_cb_gemm<1>, launch_cb_gemm<2>, launch_cb_gemm<3>, launch_cb_gemm<4>, launch_cb_gemm<5>,
    launch_cb_gemm<6>, launch_cb_gemm<7>, launch_cb_gemm<8>, launch_cb_gemm<9>, launch_cb_gemm<10>,
    launch_cb_gemm<11>, launch_cb_gemm<12>, launch_cb_gemm<13>, launch_cb_gemm<14>, launch_cb_gemm<15>,
    launch_cb_gemm<16>};
const void *const kCbGemmFuncs[kMaxCbK + 1] = {
    nullptr, (const void *)cb_gemm_kernel<1>, (const void *)cb_gemm_kernel<2>, (const void *)cb_gemm_kernel<3>,
    (const void *)cb_gemm_kernel<4>, (const void *)cb_gemm_kernel<5>, (const void *)cb_gemm_kernel<6>,
    (const void *)cb_gemm_kernel<7>, (const void *)cb_gemm_kernel<8>, (const void *)cb_gemm_kernel<9>,
    (const void *)cb_gemm_kernel<10>, (const void *)cb_gemm_kernel<11>, (const void *)cb_gemm_kernel<12>,
    (const void *)cb_gemm_kernel<13>, (const void *)cb_gemm_kernel<14>, (const void *)cb_gemm_kernel<15>,
    (const void *)cb_gemm_kernel<16>};

// Source order -> tile order (the weight order lwc_gemm_dfloat11 reads):
// each thread moves 16-byte pieces (8 weights of one row), read in source order.
__global__ void tile_order_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, uint64_t rows,
                                  uint64_t cols) {
    const uint64_t pieces = rows * cols / 8, per_row = cols / 8, k_tiles = cols / kTileCols;
    for (uint64_t c = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; c < pieces;
         c += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t r = c / per_row, col = (c % per_row) * 8;
        const uint64_t pos = ((r / kTileRows) * k_tiles + col / kTileCols) * kTileElems + (r % kTileRows) * kTileCols +
                             col % kTileCols;
        dst[pos / 8] = src[c];
    }
}

// ---- host ------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct GemmDevice {
    int sms = 0;
    int max_smem = 0;
    bool ready = false;
};

std::mutex g_gemm_mutex;
std::vector<GemmDevice> g_gemm_dev;
EncodeTiledFn g_encode_tiled = nullptr;

lwc_status gemm_device(GemmDevice &out, EncodeTiledFn &encode) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
    std::lock_guard<std::mutex> lock(g_gemm_mutex);
    if (!g_encode_tiled) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (err != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
            return fail(LWC_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
        g_encode_tiled = reinterpret_cast<EncodeTiledFn>(fn);
    }
    encode = g_encode_tiled;
    if ((int)g_gemm_dev.size() <= dev) g_gemm_dev.resize(dev + 1);
    GemmDevice &c = g_gemm_dev[dev];
    if (!c.ready) {
        int major = 0;
        err = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (err == cudaSuccess && major != 10)
            return fail(LWC_ERR_UNSUPPORTED, "the tensor-core product needs an sm_100 device (compute capability %d.x)",
                        major);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&c.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute((const void *)df11_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       c.max_smem);
        for (uint32_t k = 1; k <= kMaxCbK && err == cudaSuccess; k++)
            err = cudaFuncSetAttribute(kCbGemmFuncs[k], cudaFuncAttributeMaxDynamicSharedMemorySize, c.max_smem);
        if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "device setup: %s", cudaGetErrorString(err));
        c.ready = true;
    }
    out = c;
    return LWC_OK;
}

// Work units spread over `ctas` CTAs: every unit (128 rows of one matrix)
// costs its k-tiles plus a fixed overhead; units are taken longest first and
// each goes to the least loaded CTA (ties: the lower index); each CTA then
// takes its units grouped by matrix (one table build per matrix). Returns
// false when a CTA would get more than kMaxCtaUnits units.
bool schedule_units(const std::vector<uint32_t> &units, const std::vector<uint32_t> &cost, uint32_t ctas,
                    GemmBatch &B) {
    std::vector<uint32_t> order(units.size());
    std::iota(order.begin(), order.end(), 0u);
    std::stable_sort(order.begin(), order.end(), [&](uint32_t a, uint32_t b) { return cost[a] > cost[b]; });
    // min-heap of (load, CTA): the least loaded CTA, the lower index on ties
    std::vector<std::pair<uint64_t, uint32_t>> heap;
    heap.reserve(ctas);
    for (uint32_t c = 0; c < ctas; c++) heap.push_back({0, c});
    const auto later = [](const std::pair<uint64_t, uint32_t> &a, const std::pair<uint64_t, uint32_t> &b) {
        return a > b;
    };
    std::vector<std::vector<uint16_t>> per(ctas);
    for (uint32_t j : order) {
        std::pop_heap(heap.begin(), heap.end(), later);
        auto &top = heap.back();
        per[top.second].push_back((uint16_t)units[j]);
        top.first += cost[j];
        std::push_heap(heap.begin(), heap.end(), later);
    }
    uint32_t pos = 0;
    for (uint32_t c = 0; c < ctas; c++) {
        if (per[c].size() > kMaxCtaUnits) return false;
        std::sort(per[c].begin(), per[c].end());
        B.cta_begin[c] = (uint16_t)pos;
        for (uint16_t u : per[c]) B.sched[pos++] = u;
    }
    B.cta_begin[ctas] = (uint16_t)pos;
    return true;
}

lwc_status gemm_batched(uint32_t codec, const lwc_desc *descs, const void *const *d_blobs, const uint64_t *cols,
                        const uint16_t *const *d_xs, int M, float *const *d_ys, int count, uint32_t *d_status,
                        lwc_stream_t stream) {
    if (count < 0 || (count > 0 && (!descs || !d_blobs || !cols || !d_xs || !d_ys)))
        return fail(LWC_ERR_INVALID_ARG, "bad batch arguments");
    if (count > (int)kMaxMats) return fail(LWC_ERR_UNSUPPORTED, "at most %u matrices per call", kMaxMats);
    if (M < 1 || M > (int)kMaxM) return fail(LWC_ERR_INVALID_ARG, "M must be 1..%u (got %d)", kMaxM, M);
    if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u))
        return fail(LWC_ERR_MISALIGNED, "status word must be 4-byte aligned");
    static GemmBatch B;   // large (about 12 KB): built under the lock below, copied into the launch
    static std::mutex batch_mutex;
    std::lock_guard<std::mutex> lock(batch_mutex);
    std::memset(&B, 0, sizeof B);
    std::vector<uint32_t> units, cost;
    uint64_t max_count = 0, max_tables = 0;
    uint32_t chunk_bytes = 0, n = 0, cb_k = 0;
    const bool cb = codec == LWC_CODEC_CODEBOOK;
    std::vector<int> mats;
    for (int i = 0; i < count; i++) {
        const lwc_desc &d = descs[i];
        lwc_status st = cb ? check_codebook_desc(&d) : check_df11_desc(&d);
        if (st) return st;
        if (d.n == 0) continue;
        if (cb) {
            if (d.k < 1 || d.k > kMaxCbK)
                return fail(LWC_ERR_UNSUPPORTED, "matrix %d: codebook index width %u (1..%u taken)", i, d.k, kMaxCbK);
            if (cb_k && d.k != cb_k) return fail(LWC_ERR_UNSUPPORTED, "matrices of one call must share the index width");
            cb_k = d.k;
        } else {
            if (d.elem != LWC_ELEM_BF16) return fail(LWC_ERR_UNSUPPORTED, "matrix %d: BF16 weights only", i);
            if (d.threads_per_block != 32 || !(d.flags & kFlagChunkCounts) || (d.flags & kFlagSingleExponent))
                return fail(LWC_ERR_UNSUPPORTED,
                            "matrix %d: needs blocks of 32 chunks with stored chunk counts and more than one exponent", i);
        }
        if (cols[i] == 0 || cols[i] % kTileCols || cols[i] > (1u << 24) || d.n % cols[i])
            return fail(LWC_ERR_INVALID_ARG, "matrix %d: cols must divide n and be a multiple of 64 up to 2^24", i);
        const uint64_t rows = d.n / cols[i];
        if (rows % kTileRows || rows / kTileRows > 4096)
            return fail(LWC_ERR_INVALID_ARG, "matrix %d: rows must be a multiple of 128 (at most 2^19)", i);
        if (!cb && chunk_bytes && d.chunk_bytes != chunk_bytes)
            return fail(LWC_ERR_UNSUPPORTED, "matrices of one call must share chunk_bytes");
        if (!cb) chunk_bytes = d.chunk_bytes;
        if (!d_blobs[i] || !d_xs[i] || !d_ys[i]) return fail(LWC_ERR_INVALID_ARG, "NULL device pointer (matrix %d)", i);
        if (!aligned16(d_blobs[i]) || !aligned16(d_xs[i]) || (reinterpret_cast<uintptr_t>(d_ys[i]) & 3u))
            return fail(LWC_ERR_MISALIGNED, "blob and x must be 16-byte aligned, y 4-byte aligned (matrix %d)", i);
        const uint8_t *base = static_cast<const uint8_t *>(d_blobs[i]);
        GemmMat &g = B.m[n];
        if (cb) {
            g.packed = base + d.off_packed;
            g.table = reinterpret_cast<const uint16_t *>(base + d.off_table);
            g.table_words = (d.U + 1) / 2;
        }
        if (!cb) {
        g.t.stream = reinterpret_cast<const uint32_t *>(base + d.off_stream);
        g.t.gaps = base + d.off_gaps;
        g.t.counts = base + d.off_counts;
        g.t.blkoff = reinterpret_cast<const uint64_t *>(base + d.off_blkoff);
        g.t.sm = base + d.off_sm;
        g.t.lut = reinterpret_cast<const uint16_t *>(base + d.off_lut);
        g.t.n = d.n;
        g.t.total_bits = d.total_bits;
        g.t.stream_bytes = d.stream_bytes;
        g.t.n_blocks = (uint32_t)d.n_blocks;
        g.t.n_tables = d.n_tables;
        max_count = std::max<uint64_t>(max_count, d.max_block_count);
        max_tables = std::max<uint64_t>(max_tables, d.n_tables);
        }
        g.y = d_ys[i];
        g.rows = (uint32_t)rows;
        g.cols = (uint32_t)cols[i];
        g.k_tiles = g.cols / kTileCols;
        g.kt_split = 0;
        mats.push_back(i);
        n++;
    }
    if (n == 0) {
        clear_error();
        return LWC_OK;
    }
    GemmDevice dev;
    EncodeTiledFn encode = nullptr;
    lwc_status st = gemm_device(dev, encode);
    if (st) return st;
    // Work units: 128 rows of a matrix, all k-tiles; a matrix whose unit would
    // take much longer than a CTA's average share has its K range split in
    // two parts (the CTA that finishes a part second adds the two).
    {
        uint64_t total_cost = 0, n_units = 0;
        for (uint32_t j = 0; j < n; j++) {
            total_cost += (uint64_t)(B.m[j].rows / kTileRows) * (B.m[j].k_tiles + 2);
            n_units += B.m[j].rows / kTileRows;
        }
        const uint64_t ctas0 = std::min<uint64_t>(n_units, (uint64_t)std::min(dev.sms, (int)kMaxCtas));
        for (uint32_t j = 0; j < n; j++) {
            GemmMat &g = B.m[j];
            if (g.k_tiles >= 2 && 4 * (uint64_t)(g.k_tiles + 2) * ctas0 > 3 * total_cost) g.kt_split = g.k_tiles / 2;
            for (uint32_t r = 0; r < g.rows / kTileRows; r++) {
                if (!g.kt_split) {
                    units.push_back(j << 13 | r);
                    cost.push_back(g.k_tiles + 2);
                } else {
                    units.push_back(j << 13 | r);
                    cost.push_back(g.kt_split + 2);
                    units.push_back(j << 13 | 1u << 12 | r);
                    cost.push_back(g.k_tiles - g.kt_split + 2);
                }
            }
        }
    }
    if (units.size() > kMaxUnits) return fail(LWC_ERR_UNSUPPORTED, "more than %u 128-row units in one call", kMaxUnits);
    B.count = n;
    B.M = (uint32_t)M;
    B.n_pad = (uint32_t)round_up((uint64_t)M, 16);
    B.chunk_words = chunk_bytes / 4;
    B.seg_words = (uint32_t)round_up(32ull * B.chunk_words + 2, 4);
    B.stage_bytes = (uint32_t)round_up(max_count + 16, 16);
    B.lut_entries = (uint32_t)(max_tables * 256);
    B.acc_cols = B.n_pad <= 32 ? 32 : B.n_pad <= 64 ? 64 : B.n_pad <= 128 ? 128 : 256;
    B.tmem_cols = 2 * B.acc_cols;   // two accumulators: a unit's epilogue overlaps the next unit's MMAs
    B.idesc = umma::instr_desc_bf16_f32(kTileRows, B.n_pad);
    B.status = d_status;
    // decoder warps: at most as many as keep about kInFlightWeights weights in flight
    // (blocks of 36-byte chunks, ~3,600 weights: 12 warps; of 20-byte chunks: 20);
    // then, by shared memory, the most of them with at least three weight stages
    // (and as many stages as fit, up to kMaxStages); failing that, with two
    uint32_t warp_cap = (uint32_t)std::min<uint64_t>(kMaxDecWarps, kInFlightWeights / std::max<uint64_t>(max_count, 1));
    warp_cap = cb ? kMaxCbDecWarps : std::max(kMinDecWarps, warp_cap & ~1u);   // codebook tasks hold 1024 weights
    uint64_t smem = 0;
    auto fits = [&](uint32_t warps, uint32_t stages) {
        smem = GemmLayout(B.n_pad, stages, B.seg_words, B.lut_entries, B.stage_bytes, warps, cb_k).total + 1024;
        return smem <= (uint64_t)dev.max_smem;
    };
    B.stages = 0;
    for (uint32_t min_stages : {3u, 2u}) {
        for (uint32_t w = warp_cap; w >= kMinDecWarps && !B.stages; w -= 2)
            if (fits(w, min_stages)) {
                B.dec_warps = w;
                B.stages = min_stages;
                while (B.stages < kMaxStages && fits(w, B.stages + 1)) B.stages++;
            }
        if (B.stages) break;
    }
    if (!B.stages)
        return fail(LWC_ERR_UNSUPPORTED, "the tensor-core product does not fit in shared memory for M = %d", M);
    fits(B.dec_warps, B.stages);   // smem of the choice
    for (uint32_t j = 0; j < n; j++) {
        const int i = mats[j];
        const cuuint64_t gdim[2] = {cols[i], (cuuint64_t)M};
        const cuuint64_t gstride[1] = {cols[i] * 2};
        const cuuint32_t box[2] = {kTileCols, B.n_pad};
        const cuuint32_t estride[2] = {1, 1};
        const CUresult r = encode(&B.xmap[j], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(d_xs[i]), gdim,
                                  gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(LWC_ERR_CUDA, "tensor map of x (matrix %d): driver error %d", i, (int)r);
    }
    const uint32_t ctas = (uint32_t)std::min<uint64_t>(units.size(), (uint64_t)std::min(dev.sms, (int)kMaxCtas));
    if (!schedule_units(units, cost, ctas, B))
        return fail(LWC_ERR_UNSUPPORTED, "too many units per CTA (%zu units on %u CTAs)", units.size(), ctas);
    for (uint32_t j = 0; j < n; j++)
        if (B.m[j].kt_split) {
            const cudaError_t e = cudaMemsetAsync(B.m[j].y, 0xFF, (size_t)M * B.m[j].rows * sizeof(float),
                                                  reinterpret_cast<cudaStream_t>(stream));
            if (e != cudaSuccess) return fail(LWC_ERR_CUDA, "output fill: %s", cudaGetErrorString(e));
        }
    const dim3 grid(ctas), block((kDec0 + B.dec_warps) * 32u);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cb)
        kCbGemmKernels[cb_k](B, grid, block, (size_t)smem, s);
    else
        df11_gemm_kernel<<<grid, block, (size_t)smem, s>>>(B);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "tensor-core product launch: %s", cudaGetErrorString(err));
    clear_error();
    return LWC_OK;
}

}  // namespace
}  // namespace lwc

using namespace lwc;

extern "C" {

lwc_status lwc_tile_order(const uint16_t *d_src, uint64_t rows, uint64_t cols, uint16_t *d_dst, lwc_stream_t stream) {
    if (rows % kTileRows || cols % kTileCols)
        return fail(LWC_ERR_INVALID_ARG, "rows must be a multiple of 128 and cols of 64 (got %llu x %llu)",
                    (unsigned long long)rows, (unsigned long long)cols);
    if (rows == 0 || cols == 0) {
        clear_error();
        return LWC_OK;
    }
    if (!d_src || !d_dst) return fail(LWC_ERR_INVALID_ARG, "NULL device pointer");
    if (d_src == d_dst) return fail(LWC_ERR_INVALID_ARG, "the tile order is not computed in place");
    if (!aligned16(d_src) || !aligned16(d_dst)) return fail(LWC_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
    if (rows > (1ull << 40) / cols) return fail(LWC_ERR_INVALID_ARG, "matrix too large");
    int dev = 0, sms = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "device query: %s", cudaGetErrorString(err));
    const uint64_t pieces = rows * cols / 8;
    const uint64_t grid = std::min<uint64_t>((pieces + 255) / 256, (uint64_t)sms * 8);
    tile_order_kernel<<<(unsigned)grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint4 *>(d_src), reinterpret_cast<uint4 *>(d_dst), rows, cols);
    err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "tile-order launch: %s", cudaGetErrorString(err));
    clear_error();
    return LWC_OK;
}

lwc_status lwc_gemm_dfloat11_batched(const lwc_desc *descs, const void *const *d_blobs, const uint64_t *cols,
                                     const uint16_t *const *d_xs, int M, float *const *d_ys, int count,
                                     uint32_t *d_status, lwc_stream_t stream) {
    return gemm_batched(LWC_CODEC_DFLOAT11, descs, d_blobs, cols, d_xs, M, d_ys, count, d_status, stream);
}

lwc_status lwc_gemm_codebook_batched(const lwc_desc *descs, const void *const *d_blobs, const uint64_t *cols,
                                     const uint16_t *const *d_xs, int M, float *const *d_ys, int count,
                                     uint32_t *d_status, lwc_stream_t stream) {
    return gemm_batched(LWC_CODEC_CODEBOOK, descs, d_blobs, cols, d_xs, M, d_ys, count, d_status, stream);
}

lwc_status lwc_gemm_codebook(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x, int M,
                             float *d_y, uint32_t *d_status, lwc_stream_t stream) {
    if (!desc) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    return lwc_gemm_codebook_batched(desc, &d_blob, &cols, &d_x, M, &d_y, 1, d_status, stream);
}

lwc_status lwc_gemm_dfloat11(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x, int M,
                             float *d_y, uint32_t *d_status, lwc_stream_t stream) {
    if (!desc) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    return lwc_gemm_dfloat11_batched(desc, &d_blob, &cols, &d_x, M, &d_y, 1, d_status, stream);
}

}  // extern "C"
