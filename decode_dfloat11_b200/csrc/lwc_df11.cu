// DFloat11-style decoder for sm_100a.
//
// What it computes ("Koniec z kompromisami! DFloat11 ratuje dokładność modeli
// AI ...", section "Przełom: DFloat11 – bezstratna kompresja z wydajnością
// GPU"): every weight is rebuilt from its Huffman-coded 8-bit exponent and its
// raw sign|mantissa byte, bit for bit.
//
// How (same page, section "Jak to działa w praktyce? Magia na poziomie GPU"):
//  * small linked lookup tables held in shared memory: the blob's
//    hierarchical 256-entry tables (one per 8 code bits), fronted by three
//    2048-entry tables this kernel builds from them (symbols, code-end masks,
//    code counts), which resolve every code that fits in the next 11 stream
//    bits: several codes per lookup;
//  * two phases: each thread counts the codes that start in its chunk of the
//    stream, a scan turns the counts into output positions, and the threads
//    decode again, this time writing exponents to a shared-memory staging
//    buffer; the staged exponents are then merged with the sign|mantissa
//    bytes (and, for FP32 / FP16 elements, the raw low mantissa bits) and
//    written out with 16-byte stores. Both passes take two table entries per
//    32-bit window (up to 22 bits per step);
//  * all matrices of a transformer block in one launch: the grid walks a work
//    list of (tensor, block) items; CTAs are persistent, take contiguous runs
//    of items and rebuild their tables only when the tensor changes.
// Blocks never wait on one another: each block's first output index is stored
// in the blob, so there is no inter-block scan.
//
// Two kernels. df11_warp_kernel (blocks of 32 chunks, the encoder's default):
// one warp decodes one block with a warp scan and its own segment buffer,
// staging area and mbarrier, so no CTA-wide barrier sits on the per-block
// path; 18 warps per CTA share the tables. df11_decode_kernel (blocks of 64+
// chunks): one block per CTA and a block scan. Blobs that store each chunk's
// code count take df11_counted_kernel (the first phase read, not recomputed);
// its instance for codes of at most 8 bits also decodes codes whose words all
// have one length straight from the weight index (decode_fixed_range).
//
// Memory pipeline: as soon as pass 2 of an item no longer needs the shared
// stream segment, the bulk-copy (TMA) engine starts bringing in the segment
// and chunk gaps of the next item, overlapping the merge; the sign|mantissa
// bytes are loaded into registers at the start of an item, under both decode
// passes; block offsets are loaded one item ahead. No wait is unbounded.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "lwc_device.cuh"
#include "lwc_df11_dev.cuh"
#include "lwc_internal.h"

namespace lwc {
namespace {

using namespace df11dev;

constexpr int kMaxBatch = 32;
// symbol table (u32) + end-mask table (u16) + count table (u8)
constexpr uint32_t kFastBytes = kFastSize * (4 + 2 + 1);
constexpr int kMergeRegs = 6;   // 16-weight groups per thread whose loads are issued early
constexpr int kCtasPerSm = 4;   // target residency for 256-thread CTAs (shared memory sized for it)

struct Df11Batch {
    Df11Tensor t[kMaxBatch];
    uint32_t count;
    uint32_t total_work;
    uint32_t chunk_words;  // chunk_bytes / 4
    uint32_t seg_words;    // words staged per block: T * chunk_words + 2, rounded up to 4
    uint32_t stage_bytes;  // exponent staging capacity (>= max_block_count + 16)
    uint32_t lut_entries;  // lookup-table entries reserved in shared memory
    uint32_t warps;        // per-warp kernel: warps per CTA (fewer than kWarpsPerCta for large chunks)
    uint32_t *status;
};

// Shared-memory layout of one CTA (T threads); every offset a multiple of 16.
struct Layout {
    uint32_t lut, bufs, buf_bytes, stage, sums, bars, total;
    __host__ __device__ Layout(uint32_t T, uint32_t seg_words, uint32_t lut_entries, uint32_t stage_bytes) {
        lut = kFastBytes;
        bufs = lut + 2 * lut_entries;
        buf_bytes = 4 * seg_words + T + 16;   // segment words, then the block's T gap bytes + the next one
        stage = bufs + buf_bytes;
        sums = stage + stage_bytes;
        bars = sums + 128;
        total = bars + 16;
    }
};

// ---- lookup tables ---------------------------------------------------------

// Fast tables, indexed by the next kFastBits (11) stream bits:
//  cnt_tab[v]  = count << 4 | bits, for all whole codes inside the window
//                (entries are summed: the sum of the `bits` parts is known, so
//                one add per lookup counts codes);
//  mask_tab[v] = bit (e - 1) set for every whole code that ends e bits in;
//  sym_tab[v]  = sym0 | sym1 << 8 | sym2 << 16 | n << 24 | bits << 26, for the
//                first n <= 3 of them.
// Zero count/symbol entries mean "the first code is longer than the window".
__device__ void build_fast_tables(const uint16_t *lut, uint32_t ntab, uint8_t *cnt_tab, uint16_t *mask_tab,
                                  uint32_t *sym_tab) {
    for (uint32_t v = threadIdx.x; v < kFastSize; v += blockDim.x) {
        uint32_t w = v << (32 - kFastBits);
        uint32_t used = 0, cnt = 0, syms = 0, n3 = 0, used3 = 0, mask = 0, ignore = 0;
        while (cnt < (uint32_t)kFastBits) {
            const uint32_t r = lut_walk(lut, ntab, w, ignore);
            const uint32_t len = r >> 8;
            if (ignore || used + len > (uint32_t)kFastBits) break;
            if (cnt < 3) {
                syms |= (r & 0xFFu) << (8 * cnt);
                n3 = cnt + 1;
                used3 = used + len;
            }
            cnt++;
            used += len;
            mask |= 1u << (used - 1);
            w <<= len;
        }
        cnt_tab[v] = cnt ? (uint8_t)((cnt << 4) | used) : (uint8_t)0;
        mask_tab[v] = (uint16_t)mask;
        sym_tab[v] = n3 ? (syms | (n3 << 24) | (used3 << 26)) : 0u;
    }
}

// The 32 stream bits starting at bit `pos` of the staged segment (MSB first),
// keeping the last two words read: a decode step consumes at most 32 bits, so
// the word index advances by 0 or 1 per step and one shared-memory load per
// step suffices.
struct Window {
    uint32_t wi, w0, w1;
    __device__ __forceinline__ Window(const uint32_t *seg, uint32_t pos) : wi((pos >> 5) - 1u), w0(0), w1(seg[pos >> 5]) {}
    __device__ __forceinline__ uint32_t at(const uint32_t *seg, uint32_t pos) {
        const uint32_t ni = pos >> 5;
        w0 = ni != wi ? w1 : w0;
        w1 = seg[ni + 1];
        wi = ni;
        return __funnelshift_l(w1, w0, pos);
    }
};

// ---- merge ---------------------------------------------------------------------

__device__ __forceinline__ uint16_t merge1(uint32_t s, uint32_t e) {
    return (uint16_t)(((s & 0x80u) << 8) | (e << 7) | (s & 0x7Fu));
}

// Four weights from four sign|mantissa bytes s and four exponents e: a BF16
// weight's low byte is (s & 0x7F) | (e & 1) << 7 and its high byte is
// (e >> 1) | (s & 0x80), computed for four lanes of a word at once, then
// interleaved into two words of output.
__device__ __forceinline__ void merge4(uint32_t s, uint32_t e, uint32_t &w01, uint32_t &w23) {
    const uint32_t lo = (s & 0x7F7F7F7Fu) | ((e << 7) & 0x80808080u);
    const uint32_t hi = ((e >> 1) & 0x7F7F7F7Fu) | (s & 0x80808080u);
    w01 = __byte_perm(lo, hi, 0x5140u);
    w23 = __byte_perm(lo, hi, 0x7362u);
}

__device__ __forceinline__ void merge16(const uint4 &s, const uint4 &e, uint16_t *dst) {
    uint4 r0, r1;
    merge4(s.x, e.x, r0.x, r0.y);
    merge4(s.y, e.y, r0.z, r0.w);
    merge4(s.z, e.z, r1.x, r1.y);
    merge4(s.w, e.w, r1.z, r1.w);
    reinterpret_cast<uint4 *>(dst)[0] = r0;
    reinterpret_cast<uint4 *>(dst)[1] = r1;
}

// ---- other element types -----------------------------------------------------------
//
// FP32 and FP16 blobs code a BF16-shaped 16-bit pattern per element (sign,
// exponent field, top 7 mantissa bits), decoded exactly like BF16, plus raw
// low mantissa bits in the "lo" section. The merge turns the BF16-shaped
// pattern v into the element:
//   FP32: (v << 16) | lo16[i]
//   FP16: (v & 0x8000) | ((v & 0x0FFF) << 3) | lo3[i]   (exponent field < 32)

// Two FP16 elements from a word of two BF16-shaped patterns and their 3-bit tails.
__device__ __forceinline__ uint32_t fp16_pair(uint32_t v2, uint32_t lo_pair) {
    return (v2 & 0x80008000u) | ((v2 & 0x0FFF0FFFu) << 3) | lo_pair;
}

// 16 elements starting at element offset r of `out` (typed by E). FP32: their
// low halves are at lo + 2 r. FP16: `lo` is the section start (4-byte
// aligned) and the group's 48 tail bits start at byte 6 (g0 + r / 16).
// (ROT: the exponents are rotated, see merge4r.)
template <int E, bool ROT = false, typename I>
__device__ __forceinline__ void merge_group(const uint4 &s, const uint4 &e, void *out, const uint8_t *lo, I r,
                                            uint64_t g0 = 0) {
    if constexpr (E == LWC_ELEM_BF16 && !ROT) {
        merge16(s, e, static_cast<uint16_t *>(out) + r);
    } else {
        uint4 r0, r1;
        if constexpr (ROT) {
            merge4r(s.x, e.x, r0.x, r0.y);
            merge4r(s.y, e.y, r0.z, r0.w);
            merge4r(s.z, e.z, r1.x, r1.y);
            merge4r(s.w, e.w, r1.z, r1.w);
        } else {
            merge4(s.x, e.x, r0.x, r0.y);
            merge4(s.y, e.y, r0.z, r0.w);
            merge4(s.z, e.z, r1.x, r1.y);
            merge4(s.w, e.w, r1.z, r1.w);
        }
        if constexpr (E == LWC_ELEM_BF16) {
            reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + r)[0] = r0;
            reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + r)[1] = r1;
        } else if constexpr (E == LWC_ELEM_FP32) {
            const uint4 *lp = reinterpret_cast<const uint4 *>(lo + 2 * r);
            const uint4 l0 = __ldg(lp), l1 = __ldg(lp + 1);
            uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint32_t *>(out) + r);
            o[0] = make_uint4(__byte_perm(l0.x, r0.x, 0x5410u), __byte_perm(l0.x, r0.x, 0x7632u),
                              __byte_perm(l0.y, r0.y, 0x5410u), __byte_perm(l0.y, r0.y, 0x7632u));
            o[1] = make_uint4(__byte_perm(l0.z, r0.z, 0x5410u), __byte_perm(l0.z, r0.z, 0x7632u),
                              __byte_perm(l0.w, r0.w, 0x5410u), __byte_perm(l0.w, r0.w, 0x7632u));
            o[2] = make_uint4(__byte_perm(l1.x, r1.x, 0x5410u), __byte_perm(l1.x, r1.x, 0x7632u),
                              __byte_perm(l1.y, r1.y, 0x5410u), __byte_perm(l1.y, r1.y, 0x7632u));
            o[3] = make_uint4(__byte_perm(l1.z, r1.z, 0x5410u), __byte_perm(l1.z, r1.z, 0x7632u),
                              __byte_perm(l1.w, r1.w, 0x5410u), __byte_perm(l1.w, r1.w, 0x7632u));
        } else {
            // the group's 48 tail bits start at an even byte; read the aligned 8 bytes around them
            const uint64_t b0 = 6 * (g0 + r / 16);
            const uint32_t *wp = reinterpret_cast<const uint32_t *>(lo + (b0 & ~3ull));
            const uint64_t L = ((static_cast<uint64_t>(__ldg(wp + 1)) << 32) | __ldg(wp)) >> (8u * (uint32_t)(b0 & 3));
            uint32_t t[8];
#pragma unroll
            for (int j = 0; j < 8; j++)
                t[j] = (uint32_t)((L >> (6 * j)) & 7u) | ((uint32_t)((L >> (6 * j + 3)) & 7u) << 16);
            uint4 *o = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + r);
            o[0] = make_uint4(fp16_pair(r0.x, t[0]), fp16_pair(r0.y, t[1]), fp16_pair(r0.z, t[2]), fp16_pair(r0.w, t[3]));
            o[1] = make_uint4(fp16_pair(r1.x, t[4]), fp16_pair(r1.y, t[5]), fp16_pair(r1.z, t[6]), fp16_pair(r1.w, t[7]));
        }
    }
}

// One element i from its sign|mantissa byte s and exponent e (rotated if ROT).
template <int E, bool ROT = false>
__device__ __forceinline__ void merge_one(uint32_t s, uint32_t e, void *out, const uint8_t *lo, uint64_t i) {
    const uint32_t v = merge1(s, ROT ? ((e << 1) | (e >> 7)) & 0xFFu : e);
    if constexpr (E == LWC_ELEM_BF16) {
        static_cast<uint16_t *>(out)[i] = (uint16_t)v;
    } else if constexpr (E == LWC_ELEM_FP32) {
        static_cast<uint32_t *>(out)[i] = (v << 16) | reinterpret_cast<const uint16_t *>(lo)[i];
    } else {
        const uint64_t b = 3 * i;   // lo has slack bytes after the last tail
        const uint32_t t = ((uint32_t)lo[b >> 3] | ((uint32_t)lo[(b >> 3) + 1] << 8)) >> (b & 7);
        static_cast<uint16_t *>(out)[i] = (uint16_t)((v & 0x8000u) | ((v & 0x0FFFu) << 3) | (t & 7u));
    }
}

// ---- fixed-length codes ------------------------------------------------------------
//
// When every code word has one length L, code i is stream bits [i L, i L + L)
// (the stream is the codes back to back from bit 0), so weights are decoded
// straight from their index: no block offsets, gaps or counts are needed
// beyond the range a CTA owns.

// Code word c (0 <= c < 32) of a 32-weight piece whose stream bits start at a
// multiple of 32 in the words w[0..L] (MSB first).
template <int L>
__device__ __forceinline__ uint32_t fixed_field(const uint32_t (&w)[L + 1], int c) {
    const int p = c * L, k = p >> 5, o = p & 31;
    if (o + L <= 32) return (w[k] << o) >> (32 - L);
    return __funnelshift_l(w[k + 1], w[k], (uint32_t)o) >> (32 - L);
}

// The stream words (w[0..L-1], w[L] = 0) and sign|mantissa bytes of the
// 32-weight piece at weight g (a multiple of 32).
template <int L>
__device__ __forceinline__ void fixed_load(const Df11Tensor &tn, uint64_t nwords, uint64_t g, uint32_t (&w)[L + 1],
                                           uint4 &s0, uint4 &s1) {
    const uint64_t w0 = g / 32 * L;   // the piece's first stream word
    if (L % 4 == 0 && w0 + L <= nwords) {   // 16-byte aligned: w0 is a multiple of L
#pragma unroll
        for (int j = 0; j < L; j += 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(tn.stream + w0 + j));
            w[j] = v.x;
            w[j + 1] = v.y;
            w[j + 2] = v.z;
            w[j + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < L; j++) w[j] = w0 + j < nwords ? __ldg(tn.stream + w0 + j) : 0u;
    }
    w[L] = 0;
    s0 = __ldg(reinterpret_cast<const uint4 *>(tn.sm + g));
    s1 = __ldg(reinterpret_cast<const uint4 *>(tn.sm + g + 16));
}

// Decodes and merges the piece at weight g (see decode_fixed_range).
template <int E, int L, bool AFF>
__device__ __forceinline__ void fixed_emit(const Df11Tensor &tn, const uint32_t *tab, uint32_t base4, uint64_t g,
                                           const uint32_t (&w)[L + 1], const uint4 &s0, const uint4 &s1) {
    uint32_t e[8];
#pragma unroll
    for (int q = 0; q < 8; q++) {
        if constexpr (AFF && L == 8) {   // four whole bytes, first code in the top one
            e[q] = __byte_perm(w[q], 0u, 0x0123u) + base4;
        } else if constexpr (AFF) {   // each byte stays <= 255: base + 2^L - 1 <= 255
            e[q] = (fixed_field<L>(w, 4 * q) | (fixed_field<L>(w, 4 * q + 1) << 8) |
                    (fixed_field<L>(w, 4 * q + 2) << 16) | (fixed_field<L>(w, 4 * q + 3) << 24)) + base4;
        } else {
            e[q] = tab[fixed_field<L>(w, 4 * q)] | (tab[fixed_field<L>(w, 4 * q + 1)] << 8) |
                   (tab[fixed_field<L>(w, 4 * q + 2)] << 16) | (tab[fixed_field<L>(w, 4 * q + 3)] << 24);
        }
    }
    merge_group<E, !AFF>(s0, make_uint4(e[0], e[1], e[2], e[3]), tn.out, tn.lo, g);
    merge_group<E, !AFF>(s1, make_uint4(e[4], e[5], e[6], e[7]), tn.out, tn.lo, g + 16);
}

// The CTA's threads t = 0 .. nt - 1: weights [ob, oe) of tensor tn, whose
// code words all have length L (1..8); tab[v] = rotated exponent of code
// word v. AFF: code word v stands for exponent base + v (a flat histogram over
// consecutive exponents gives this canonical code), so a piece's exponents
// are its fields plus base, with no lookups. Threads take 32-weight pieces in
// turn (32 L stream bits = L words, 32 sign|mantissa bytes, two 16-weight
// merges), lane 0 of each warp bringing the warp's pieces of the next turn
// into L2; then the up to 31 weights at either end one by one. Stream reads
// stay inside the stream section whatever the offsets say; the caller
// checks ob <= oe <= n.
template <int E, int L, bool AFF>
__device__ __noinline__ void decode_fixed_range(const Df11Tensor &tn, const uint32_t *tab, uint32_t base,
                                                uint64_t ob, uint64_t oe, uint32_t t, uint32_t nt) {
    const uint64_t nwords = tn.stream_bytes >> 2;
    const uint64_t p_lo = (ob + 31) & ~31ull, p_hi = oe & ~31ull;
    const uint32_t base4 = base * 0x01010101u;
    for (uint64_t g = p_lo + 32ull * t; g < p_hi; g += 32ull * nt) {
        if ((t & 31u) == 0) {   // the warp's 1,024 weights of the next turn into L2
            const uint64_t ga = g + 32ull * nt;
            if (ga + 1024 <= p_hi) {
                dev::prefetch_l2(tn.sm + ga, 1024u);
                const uint64_t s0 = (ga / 32 * L * 4) & ~15ull, s1 = ((ga + 1024) / 32 * L * 4 + 15) & ~15ull;
                if (s1 <= (tn.stream_bytes & ~15ull))
                    dev::prefetch_l2(reinterpret_cast<const uint8_t *>(tn.stream) + s0, (uint32_t)(s1 - s0));
            }
        }
        uint32_t w[L + 1];
        uint4 s0, s1;
        fixed_load<L>(tn, nwords, g, w, s0, s1);
        fixed_emit<E, L, AFF>(tn, tab, base4, g, w, s0, s1);
    }
    // the weights before the first piece (u = 0..30) and after the last (u = 31..61)
    for (uint32_t u = t; u < 62; u += nt) {
        const uint64_t i = u < 31 ? ob + u : (p_hi > p_lo ? p_hi : p_lo) + (u - 31);
        const bool one = u < 31 ? i < (p_lo < oe ? p_lo : oe) : i < oe;
        if (one) {
            const uint64_t p = i * L, k = p >> 5;
            const uint32_t w_a = k < nwords ? __ldg(tn.stream + k) : 0u;
            const uint32_t w_b = k + 1 < nwords ? __ldg(tn.stream + k + 1) : 0u;
            const uint32_t f = __funnelshift_l(w_b, w_a, (uint32_t)p & 31u) >> (32 - L);
            merge_one<E, true>(tn.sm[i], tab[f], tn.out, tn.lo, i);
        }
    }
}

// mode = L | kFixedAffine (or not), from fixed_code_length.
template <int E>
__device__ __forceinline__ void decode_fixed(uint32_t mode, const Df11Tensor &tn, const uint32_t *tab, uint64_t ob,
                                             uint64_t oe, uint32_t t, uint32_t nt) {
    const uint32_t base = ((tab[0] << 1) | (tab[0] >> 7)) & 0xFFu;   // exponent of code word 0
    switch (mode) {
#define LWC_FIXED_CASE(L_)                                                       \
    case L_: decode_fixed_range<E, L_, false>(tn, tab, base, ob, oe, t, nt); break; \
    case L_ | kFixedAffine: decode_fixed_range<E, L_, true>(tn, tab, base, ob, oe, t, nt); break;
        LWC_FIXED_CASE(1)
        LWC_FIXED_CASE(2)
        LWC_FIXED_CASE(3)
        LWC_FIXED_CASE(4)
        LWC_FIXED_CASE(5)
        LWC_FIXED_CASE(6)
        LWC_FIXED_CASE(7)
        LWC_FIXED_CASE(8)
#undef LWC_FIXED_CASE
    default: break;
    }
}

// ---- block scan ------------------------------------------------------------------

__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_sums, uint32_t &total) {
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= (uint32_t)o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < nwarps ? warp_sums[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, s, o);
            if (lane >= (uint32_t)o) s += y;
        }
        if (lane < nwarps) warp_sums[lane] = s;
    }
    __syncthreads();
    total = warp_sums[nwarps - 1];
    const uint32_t before = warp ? warp_sums[warp - 1] : 0u;
    return before + x - v;
}

// ---- work list ----------------------------------------------------------------------

// Advance ti (monotonically) to the tensor that owns work item w.
__device__ __forceinline__ uint32_t locate(const Df11Batch &B, uint32_t w, uint32_t ti) {
    while (ti + 1 < B.count && w >= B.t[ti + 1].first_work) ++ti;
    return ti;
}

// Thread 0: start the bulk copies of item (ti, b) into buffer `buf`: the
// block's stream segment, its T chunk gaps and (when there is a next block)
// the next block's first gap, which bounds this block's last chunk.
__device__ __forceinline__ void issue_item(const Df11Batch &B, uint32_t ti, uint32_t b, uint8_t *buf,
                                           uint32_t seg_bytes, uint64_t *bar) {
    const Df11Tensor &tn = B.t[ti];
    const uint32_t T = blockDim.x;
    const uint64_t seg0 = (uint64_t)b * T * B.chunk_words * 4;   // byte offset, multiple of 128
    const uint64_t avail = tn.stream_bytes > seg0 ? tn.stream_bytes - seg0 : 0;
    const uint32_t bytes = (uint32_t)(avail < seg_bytes ? avail : seg_bytes);
    const uint32_t gbytes = b + 1 < tn.n_blocks ? T + 16 : T;
    dev::mbar_arrive_expect_tx(bar, bytes + gbytes);
    if (bytes) dev::bulk_g2s(buf, reinterpret_cast<const uint8_t *>(tn.stream) + seg0, bytes, bar);
    dev::bulk_g2s(buf + seg_bytes, tn.gaps + (uint64_t)b * T, gbytes, bar);
}

// ---- the kernel -------------------------------------------------------------------

template <int kMaxThreads, int E>
__global__ void __launch_bounds__(kMaxThreads, kCtasPerSm * 256 / kMaxThreads > 0 ? kCtasPerSm * 256 / kMaxThreads : 1)
    df11_decode_kernel(const __grid_constant__ Df11Batch B) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t T = blockDim.x, tid = threadIdx.x;
    const Layout L(T, B.seg_words, B.lut_entries, B.stage_bytes);
    uint32_t *sym_tab = reinterpret_cast<uint32_t *>(smem);
    uint16_t *mask_tab = reinterpret_cast<uint16_t *>(smem + kFastSize * 4);
    uint8_t *cnt_tab = smem + kFastSize * 6;
    uint16_t *lut = reinterpret_cast<uint16_t *>(smem + L.lut);
    uint8_t *stage = smem + L.stage;
    uint32_t *warp_sums = reinterpret_cast<uint32_t *>(smem + L.sums);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    const uint32_t seg_bytes = 4 * B.seg_words;

    const uint32_t CW = B.chunk_words, cbits = CW * 32u;
    const uint32_t W = B.total_work, G = gridDim.x;
    const uint32_t w_begin = (uint32_t)((uint64_t)W * blockIdx.x / G);
    const uint32_t w_end = (uint32_t)((uint64_t)W * (blockIdx.x + 1) / G);
    if (w_begin >= w_end) return;

    uint32_t ti = locate(B, w_begin, 0);
    if (tid == 0) {
        dev::mbar_init(&bars[0], 1);
        dev::fence_mbar_init();
        issue_item(B, ti, w_begin - B.t[ti].first_work, smem + L.bufs, seg_bytes, &bars[0]);
    }

    // block offsets of the first item; later items' are loaded one item ahead
    uint64_t o0n = B.t[ti].blkoff[w_begin - B.t[ti].first_work];
    uint64_t o1n = B.t[ti].blkoff[w_begin - B.t[ti].first_work + 1];
    uint32_t bad = 0;
    int cur = -1;
    for (uint32_t w = w_begin; w < w_end; ++w) {
        const uint32_t it = w - w_begin;
        ti = locate(B, w, ti);
        const Df11Tensor &tn = B.t[ti];
        const uint32_t b = w - tn.first_work;
        const uint64_t o0 = o0n, o1 = o1n;
        if (w + 1 < w_end) {
            const uint32_t t1 = locate(B, w + 1, ti);
            const uint32_t b1 = w + 1 - B.t[t1].first_work;
            o0n = B.t[t1].blkoff[b1];
            o1n = B.t[t1].blkoff[b1 + 1];
        }
        const bool ok = o0 <= o1 && o1 <= tn.n && o1 - o0 + 16 <= B.stage_bytes;

        // sign|mantissa bytes of this thread's first merge groups: loads
        // issued now, consumed after both decode passes
        const uint64_t g_lo = (o0 + 15) & ~15ull, g_hi = o1 & ~15ull;
        uint4 sv[kMergeRegs];
#pragma unroll
        for (int m = 0; m < kMergeRegs; m++) {
            const uint64_t g = g_lo + 16ull * (tid + (uint32_t)m * T);
            sv[m] = (ok && g < g_hi) ? __ldg(reinterpret_cast<const uint4 *>(tn.sm + g)) : make_uint4(0, 0, 0, 0);
        }

        if ((int)ti != cur) {
            // new tensor: stage its hierarchical tables, build the fast tables
            __syncthreads();
            const uint32_t nt = min(tn.n_tables, B.lut_entries / 256u);
            for (uint32_t i = tid; i < nt * 128u; i += T)
                reinterpret_cast<uint32_t *>(lut)[i] = reinterpret_cast<const uint32_t *>(tn.lut)[i];
            __syncthreads();
            build_fast_tables(lut, nt, cnt_tab, mask_tab, sym_tab);
            cur = (int)ti;
        }
        const uint32_t ntab = min(tn.n_tables, B.lut_entries / 256u);

        // this item's segment and gaps (its copy is the only one in flight)
        const bool arrived = dev::mbar_wait_bounded(&bars[0], it & 1u);
        if (__syncthreads_or(!arrived)) {
            // let the late copy land (bounded) before the CTA's shared memory goes away
            bad |= LWC_DEVICE_TIMEOUT;
            if (tid == 0) dev::mbar_wait_bounded(&bars[0], it & 1u);
            break;
        }
        bool next_issued = false;
        const uint8_t *buf = smem + L.bufs;
        const uint32_t *seg = reinterpret_cast<const uint32_t *>(buf);

        if (ok) {
            // this thread decodes the codes in [start, end): from its chunk's
            // first code to the next chunk's first code (or the stream end),
            // so the range holds whole codes only
            const uint64_t rem_block = tn.total_bits - (uint64_t)b * T * cbits;
            const uint32_t start = tid * cbits + buf[seg_bytes + tid];
            const bool has_next = tid + 1 < T || b + 1 < tn.n_blocks;
            const uint64_t next = has_next ? (uint64_t)(tid + 1) * cbits + buf[seg_bytes + tid + 1] : rem_block;
            const uint32_t end = (uint32_t)min(next, rem_block);

            // phase 1: count the codes in [start, end)
            uint32_t count = 0;
            if (start < end) {
                uint32_t pos = start, rem = end - start, acc = 0, sbits = 0, scount = 0;
                Window win(seg, start);
                for (;;) {
                    const uint32_t wv = win.at(seg, pos);
                    const uint32_t idx = wv >> (32 - kFastBits);
                    const uint32_t e = cnt_tab[idx];
                    const uint32_t len = e & 15u;
                    // two entries from one 32-bit window (the first takes at most 11 bits)
                    const uint32_t e2 = cnt_tab[(wv << len) >> (32 - kFastBits)];
                    const uint32_t l2 = e2 & 15u;
                    if ((len - 1u < rem) & (l2 - 1u < rem - len)) {
                        acc += e + e2;
                        pos += len + l2;
                        rem -= len + l2;
                        continue;
                    }
                    if (len - 1u < rem) {   // whole entry inside the range (len 0: long code)
                        acc += e;
                        pos += len;
                        rem -= len;
                        continue;
                    }
                    if (rem == 0) break;
                    if (e == 0) {          // first code longer than the window
                        const uint32_t l = lut_walk(lut, ntab, wv, bad) >> 8;
                        if (l > rem) {
                            bad |= LWC_DEVICE_BAD_CODE;
                            break;
                        }
                        pos += l;
                        rem -= l;
                        sbits += l;
                        scount++;
                        continue;
                    }
                    scount += __popc(mask_tab[idx] & ((1u << rem) - 1u));   // codes ending inside the range
                    break;
                }
                count = ((acc - (pos - start - sbits)) >> 4) + scount;
            }

            uint32_t total;
            const uint32_t first = block_exclusive_scan(count, warp_sums, total);
            if (total == (uint32_t)(o1 - o0)) {
                // phase 2: decode again, writing exponents to stage[(o0 & 15) + first ...]
                if (start < end) {
                    uint8_t *bp = stage + (uint32_t)(o0 & 15u) + first;
                    uint32_t pos = start, rem = end - start;
                    Window win(seg, start);
                    for (;;) {
                        const uint32_t wv = win.at(seg, pos);
                        const uint32_t idx = wv >> (32 - kFastBits);
                        const uint32_t e = sym_tab[idx];
                        const uint32_t len = e >> 26;
                        const uint32_t e2 = sym_tab[(wv << len) >> (32 - kFastBits)];
                        const uint32_t l2 = e2 >> 26;
                        if ((len - 1u < rem) & (l2 - 1u < rem - len)) {   // two entries, one window
                            const uint32_t n = (e >> 24) & 3u, n2 = (e2 >> 24) & 3u;
                            bp[0] = (uint8_t)e;
                            if (n > 1) bp[1] = (uint8_t)(e >> 8);
                            if (n > 2) bp[2] = (uint8_t)(e >> 16);
                            uint8_t *bq = bp + n;
                            bq[0] = (uint8_t)e2;
                            if (n2 > 1) bq[1] = (uint8_t)(e2 >> 8);
                            if (n2 > 2) bq[2] = (uint8_t)(e2 >> 16);
                            bp = bq + n2;
                            pos += len + l2;
                            rem -= len + l2;
                            continue;
                        }
                        if (len - 1u < rem) {
                            const uint32_t n = (e >> 24) & 3u;
                            bp[0] = (uint8_t)e;
                            if (n > 1) bp[1] = (uint8_t)(e >> 8);
                            if (n > 2) bp[2] = (uint8_t)(e >> 16);
                            bp += n;
                            pos += len;
                            rem -= len;
                            continue;
                        }
                        if (rem == 0) break;
                        if (e == 0) {
                            const uint32_t r = lut_walk(lut, ntab, wv, bad);
                            const uint32_t l = r >> 8;
                            if (l > rem) break;
                            *bp++ = (uint8_t)r;
                            pos += l;
                            rem -= l;
                            continue;
                        }
                        const uint32_t j = __popc(mask_tab[idx] & ((1u << rem) - 1u));   // < 3
                        if (j > 0) bp[0] = (uint8_t)e;
                        if (j > 1) bp[1] = (uint8_t)(e >> 8);
                        break;
                    }
                }
                __syncthreads();
                // the segment is free: fetch the next item's while merging this one
                if (tid == 0 && w + 1 < w_end) {
                    const uint32_t t1 = locate(B, w + 1, ti);
                    dev::fence_proxy_async_smem();
                    issue_item(B, t1, w + 1 - B.t[t1].first_work, smem + L.bufs, seg_bytes, &bars[0]);
                }
                next_issued = true;

                // merge exponents with sign|mantissa bytes, 16 weights per group
                const uint64_t base = o0 & ~15ull;
#pragma unroll
                for (int m = 0; m < kMergeRegs; m++) {
                    const uint64_t g = g_lo + 16ull * (tid + (uint32_t)m * T);
                    if (g < g_hi)
                        merge_group<E>(sv[m], *reinterpret_cast<const uint4 *>(stage + (g - base)), tn.out, tn.lo, g);
                }
                for (uint64_t g = g_lo + 16ull * (tid + (uint32_t)kMergeRegs * T); g < g_hi; g += 16ull * T)
                    merge_group<E>(__ldg(reinterpret_cast<const uint4 *>(tn.sm + g)),
                                   *reinterpret_cast<const uint4 *>(stage + (g - base)), tn.out, tn.lo, g);
                if (tid < 32) {   // partial 16-groups at both ends
                    const uint64_t i = tid < 16 ? o0 + tid : max(g_hi, g_lo) + (tid - 16);
                    const bool head = tid < 16 && i < min(g_lo, o1);
                    const bool tail = tid >= 16 && i < o1;
                    if (head || tail) merge_one<E>(tn.sm[i], stage[i - base], tn.out, tn.lo, i);
                }
            } else {
                bad |= LWC_DEVICE_BAD_COUNT;   // `total` is the same in every thread
            }
        } else {
            bad |= LWC_DEVICE_BAD_OFFSET;      // same decision in every thread
        }
        __syncthreads();   // the segment and the staging area are free again

        if (tid == 0 && !next_issued && w + 1 < w_end) {   // items skipped as corrupt
            const uint32_t t1 = locate(B, w + 1, ti);
            dev::fence_proxy_async_smem();
            issue_item(B, t1, w + 1 - B.t[t1].first_work, smem + L.bufs, seg_bytes, &bars[0]);
        }
    }
    if (bad && B.status) atomicOr(B.status, bad);
}

// ---- per-warp blocks ----------------------------------------------------------------
//
// Blobs encoded with threads_per_block = 32 have one block per 32 chunks, so a
// single warp can decode a block on its own: its output offset is stored, the
// scan is a warp scan, and nothing waits for the other warps of the CTA. The
// CTA's 18 warps share the lookup tables (rebuilt, with CTA barriers, only
// where the CTA's run of blocks crosses into the next tensor); each warp has
// its own segment buffer, gap bytes, staging area and mbarrier, and walks the
// blocks w, w + 18, w + 36, ... of the current tensor (fewer warps per CTA,
// and a shorter stride, when long chunks make a warp's buffers too large for
// 18 of them).
constexpr uint32_t kWarpsPerCta = 18;   // 2 CTAs (36 warps) per SM fit registers and shared memory
constexpr int kWarpCtasPerSm = 2;
// The counted decoder's wide form: one CTA of 32 warps per SM. The SM's
// schedulers do not serve two CTAs evenly, so of two CTAs with equal shares one
// finishes early and its sibling runs the rest with half the warps; with one
// CTA every warp claims from the same counter. That outweighs the four fewer
// warps on long launches (a Llama-3-70B layer: 0.580 -> 0.572 ms; the model
// pass 2.4 % faster) but not on short ones (a Llama-3-8B layer: 0.164 -> 0.170).
constexpr uint32_t kWideWarpsPerCta = 32;
constexpr uint64_t kWideMinWeights = 512ull << 20;   // launches of at least this many weights
constexpr int kWarpMergeRegs = 3;       // 16-weight merge groups per lane whose loads are issued early

struct WarpLayout {
    uint32_t warp0, seg_bytes, stage, warp_bytes, bars, total;
    __host__ __device__ WarpLayout(uint32_t seg_words, uint32_t lut_entries, uint32_t stage_bytes, uint32_t warps) {
        warp0 = kFastBytes + ((2 * lut_entries + 15) & ~15u);
        seg_bytes = 4 * seg_words;
        stage = seg_bytes + 48;   // the block's 32 gap bytes, then the next block's first 16
        warp_bytes = stage + stage_bytes;
        bars = warp0 + warps * warp_bytes;
        total = bars + 8 * warps;
    }
};

// Lane 0: start the bulk copies of block b of tensor `tn` into this warp's buffer.
__device__ __forceinline__ void issue_warp_item(const Df11Batch &B, const Df11Tensor &tn, uint32_t b, uint8_t *buf,
                                                uint32_t seg_bytes, uint64_t *bar) {
    const uint64_t seg0 = (uint64_t)b * 32u * B.chunk_words * 4;   // multiple of 128
    const uint64_t avail = tn.stream_bytes > seg0 ? tn.stream_bytes - seg0 : 0;
    const uint32_t bytes = (uint32_t)(avail < seg_bytes ? avail : seg_bytes);
    const uint32_t gbytes = b + 1 < tn.n_blocks ? 48u : 32u;
    dev::mbar_arrive_expect_tx(bar, bytes + gbytes);
    if (bytes) dev::bulk_g2s(buf, reinterpret_cast<const uint8_t *>(tn.stream) + seg0, bytes, bar);
    dev::bulk_g2s(buf + seg_bytes, tn.gaps + (uint64_t)b * 32u, gbytes, bar);
}

// ---- fused linear layer ---------------------------------------------------------------
//
// y[m, r] = sum_c W[r, c] x[m, c] for M <= 8 activation rows: the weights a
// warp decodes into its staging area are dotted with the activations instead
// of being stored. W is rows x cols row-major, so a block's weights [o0, o1)
// end one row, span whole rows and start another. The block's weights are
// taken in rounds, in order (the single weights before its first 16-weight
// group, rounds of 32 groups, the single weights after its last group); each
// lane forms its part of a round as one FMA chain per activation row and adds
// it to its running sum for the open row; when a round reaches the next row,
// the finished row's lane sums are summed across the warp and added to y with
// one atomic add per activation row. Summation tree height per output: at
// most 16 (chain) + ceil(cols / 512) + 4 (running sum) + 5 (warp) + the number
// of blocks sharing the row (a block of 32 chunks of at least 8 bytes holds at
// least 63 codes of at most 32 bits), within ceil(cols / 512) + ceil(cols /
// 32) + 32. Rows whose length is not a multiple of 16 take one atomic add
// per weight (height cols).

constexpr int kMaxLinBatch = 16;
constexpr int kMaxRows = 8;
constexpr uint32_t kNoRow = 0xFFFFFFFFu;

struct Df11Lin {
    const uint16_t *x[kMaxLinBatch];   // M x cols BF16, row-major
    float *y[kMaxLinBatch];            // M x rows FP32, row-major, zeroed before the launch
    uint64_t rows[kMaxLinBatch];
    uint32_t cols[kMaxLinBatch];
    uint32_t magic[kMaxLinBatch];      // division by cols, see div_cols
    uint32_t shifts[kMaxLinBatch];     // sh1 | sh2 << 8
    uint32_t M;
};

// n / cols for any 32-bit n, with m' and the shifts precomputed on the host
// (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", PLDI 1994, section 4, unsigned division: t = MULUH(m', n),
// q = SRL(t + SRL(n - t, sh1), sh2)).
__device__ __forceinline__ uint32_t div_cols(uint32_t n, uint32_t magic, uint32_t shifts) {
    const uint32_t t = __umulhi(magic, n);
    return (t + ((n - t) >> (shifts & 0xFFu))) >> (shifts >> 8);
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

// Warp sums of c[m]; lane 0 adds them to y[m, row].
template <int MM>
__device__ __forceinline__ void lin_flush(const float (&c)[MM], uint32_t M, float *y, uint64_t rows,
                                          uint64_t row, uint32_t lane) {
#pragma unroll
    for (int m = 0; m < MM; m++) {
        if ((uint32_t)m < M) {
            float v = c[m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
            if (lane == 0) atomicAdd(y + (uint64_t)m * rows + row, v);
        }
    }
}

// One round: each valid lane brings p[m] for row offset lr; the round's
// weights lie in rows rf .. rl (warp-uniform, rf at or after the open row
// cur). Rows before rl are flushed; acc becomes rl's lane sums.
template <int MM>
__device__ __forceinline__ void lin_round(float (&acc)[MM], uint32_t &cur, const float (&p)[MM],
                                          bool valid, uint32_t lr, uint32_t rf, uint32_t rl, uint32_t M, float *y,
                                          uint64_t rows, uint64_t row_base, uint32_t lane) {
    if (rf == rl && rl == cur) {
#pragma unroll
        for (int m = 0; m < MM; m++) acc[m] += valid ? p[m] : 0.f;
        return;
    }
    for (uint32_t rr = cur == kNoRow ? rf : cur; rr <= rl; rr++) {
        float c[MM];
#pragma unroll
        for (int m = 0; m < MM; m++) c[m] = (valid && lr == rr ? p[m] : 0.f) + (rr == cur ? acc[m] : 0.f);
        if (rr < rl) {
            lin_flush<MM>(c, M, y, rows, row_base + rr, lane);
        } else {
#pragma unroll
            for (int m = 0; m < MM; m++) acc[m] = c[m];
        }
    }
    cur = rl;
}

// The linear layer's part of one decoded block [o0, o1) (exponents staged at
// stage[i - (o0 & ~15)], rotated as merge4r takes them if ROT; sign|mantissa
// bytes of the first groups in sv).
template <int MM, bool ROT = false>
__device__ __forceinline__ void lin_block(const Df11Lin &X, uint32_t ti, const Df11Tensor &tn, const uint8_t *stage,
                                          const uint4 (&sv)[kWarpMergeRegs], uint64_t o0, uint64_t o1,
                                          uint64_t g_lo, uint64_t g_hi, uint32_t lane) {
    const uint32_t cols = X.cols[ti], M = X.M, magic = X.magic[ti], shifts = X.shifts[ti];
    const uint64_t rows = X.rows[ti];
    const uint16_t *x = X.x[ti];
    float *y = X.y[ti];
    const uint64_t base = o0 & ~15ull;
    const uint64_t row_base = base / cols;
    const uint32_t d0 = (uint32_t)(base - row_base * cols);   // column of `base`; offsets below are from base
    const uint8_t *sb = tn.sm + base;

    if (cols & 15u) {
        // rows not made of whole 16-weight groups: one atomic add per weight
        for (uint64_t i = o0 + lane; i < o1; i += 32) {
            const uint32_t r = (uint32_t)(i - base), d = d0 + r;
            const uint32_t lr = div_cols(d, magic, shifts), col = d - lr * cols;
            const float w = bf16_lo(merge1(sb[r], ROT ? ((stage[r] << 1) | (stage[r] >> 7)) & 0xFFu : stage[r]));
            for (uint32_t m = 0; m < M; m++)
                atomicAdd(y + (uint64_t)m * rows + row_base + lr, w * bf16_lo(x[(uint64_t)m * cols + col]));
        }
        return;
    }

    float acc[MM], p[MM];
#pragma unroll
    for (int m = 0; m < MM; m++) acc[m] = 0.f;
    uint32_t cur = kNoRow;

    // single weights at block-relative offset r (valid lanes); the round spans [first, last]
    auto single = [&](uint32_t r, bool valid, uint32_t first, uint32_t last) {
        const uint32_t d = d0 + r;
        const uint32_t lr = div_cols(d, magic, shifts);
#pragma unroll
        for (int m = 0; m < MM; m++) p[m] = 0.f;
        if (valid) {
            const float w = bf16_lo(merge1(sb[r], ROT ? ((stage[r] << 1) | (stage[r] >> 7)) & 0xFFu : stage[r]));
            const uint16_t *xc = x + (d - lr * cols);
#pragma unroll
            for (int m = 0; m < MM; m++)
                if ((uint32_t)m < M) p[m] = w * bf16_lo(xc[(uint64_t)m * cols]);
        }
        lin_round<MM>(acc, cur, p, valid, lr, div_cols(d0 + first, magic, shifts), div_cols(d0 + last, magic, shifts), M,
                  y, rows, row_base, lane);
    };
    // a round of 32 groups starting at block-relative rb; this lane's group at rb + 16 lane
    const uint32_t rhi = (uint32_t)(g_hi - base);
    auto groups = [&](uint32_t rb, const uint4 &s, bool valid) {
        const uint32_t r = rb + 16u * lane, d = d0 + r;
        const uint32_t lr = div_cols(d, magic, shifts);
#pragma unroll
        for (int m = 0; m < MM; m++) p[m] = 0.f;
        if (valid) {
            const uint4 e = *reinterpret_cast<const uint4 *>(stage + r);
            uint32_t wv[8];
            if constexpr (ROT) {
                merge4r(s.x, e.x, wv[0], wv[1]);
                merge4r(s.y, e.y, wv[2], wv[3]);
                merge4r(s.z, e.z, wv[4], wv[5]);
                merge4r(s.w, e.w, wv[6], wv[7]);
            } else {
                merge4(s.x, e.x, wv[0], wv[1]);
                merge4(s.y, e.y, wv[2], wv[3]);
                merge4(s.z, e.z, wv[4], wv[5]);
                merge4(s.w, e.w, wv[6], wv[7]);
            }
            const uint4 *xc = reinterpret_cast<const uint4 *>(x + (d - lr * cols));   // 16 columns, 32-byte aligned
#pragma unroll
            for (int m = 0; m < MM; m++) {
                if ((uint32_t)m < M) {
                    const uint4 a = __ldg(xc + (uint64_t)m * (cols / 8)), b = __ldg(xc + (uint64_t)m * (cols / 8) + 1);
                    const uint32_t xa[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
                    float t = 0.f;
#pragma unroll
                    for (int j = 0; j < 8; j++) t = fma2_bf16(wv[j], xa[j], t);
                    p[m] = t;
                }
            }
        }
        const uint32_t last = min(rhi, rb + 512u) - 16u;   // the round's last group (groups never straddle rows)
        lin_round<MM>(acc, cur, p, valid, lr, div_cols(d0 + rb, magic, shifts), div_cols(d0 + last, magic, shifts), M,
                  y, rows, row_base, lane);
    };

    // weights before the first group, on lanes 0..15
    const uint64_t hend = min(g_lo, o1);
    if (hend > o0) {
        const bool valid = lane < 16 && o0 + lane < hend;
        single((uint32_t)(o0 - base) + (valid ? lane : 0u), valid, (uint32_t)(o0 - base), (uint32_t)(hend - 1 - base));
    }
    // whole groups
    const uint32_t rlo = (uint32_t)(g_lo - base);
#pragma unroll
    for (int m = 0; m < kWarpMergeRegs; m++) {
        const uint32_t rb = rlo + 512u * m;
        if (rb < rhi) groups(rb, sv[m], rb + 16u * lane < rhi);
    }
    for (uint32_t rb = rlo + 512u * kWarpMergeRegs; rb < rhi; rb += 512u) {
        const bool valid = rb + 16u * lane < rhi;
        groups(rb, valid ? __ldg(reinterpret_cast<const uint4 *>(sb + rb + 16u * lane)) : make_uint4(0, 0, 0, 0), valid);
    }
    // weights after the last group, on lanes 16..31
    const uint64_t tb = max(g_hi, g_lo);
    if (o1 > tb) {
        const bool valid = lane >= 16 && tb + (lane - 16) < o1;
        single((uint32_t)(tb - base) + (valid ? lane - 16 : 0u), valid, (uint32_t)(tb - base), (uint32_t)(o1 - 1 - base));
    }
    if (cur != kNoRow) lin_flush<MM>(acc, M, y, rows, row_base + cur, lane);
}

// Single-exponent tensors: one warp per row, lane-strided columns.
__global__ void df11_linear_const_kernel(const uint8_t *__restrict__ sm, uint32_t const_exp,
                                         const uint16_t *__restrict__ x, uint32_t M, uint64_t rows, uint32_t cols,
                                         float *__restrict__ y) {
    const uint32_t lane = threadIdx.x & 31u;
    const uint64_t warps = (uint64_t)gridDim.x * (blockDim.x / 32);
    for (uint64_t r = blockIdx.x * (uint64_t)(blockDim.x / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        float acc[kMaxRows];
#pragma unroll
        for (int m = 0; m < kMaxRows; m++) acc[m] = 0.f;
        for (uint32_t c = lane; c < cols; c += 32u) {
            const float w = bf16_lo(merge1(sm[r * cols + c], const_exp));
#pragma unroll
            for (int m = 0; m < kMaxRows; m++)
                if ((uint32_t)m < M) acc[m] = fmaf(w, bf16_lo(x[(uint64_t)m * cols + c]), acc[m]);
        }
#pragma unroll
        for (int m = 0; m < kMaxRows; m++) {
            if ((uint32_t)m < M) {
                float v = acc[m];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
                if (lane == 0) y[(uint64_t)m * rows + r] = v;
            }
        }
    }
}

__global__ void zero_f32_kernel(float *__restrict__ y, uint64_t n) {
    for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x)
        y[i] = 0.f;
}

// The per-warp decoder's body. LIN = false: store the weights (decoder).
// LIN = true: dot them with the activations instead (fused linear layer, BF16
// elements only).
template <int E, int LIN>   // LIN: 0 = decoder, else the linear layer for up to LIN activation rows
__device__ __forceinline__ void df11_warp_body(const Df11Batch &B, const Df11Lin *X) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const uint32_t NW = B.warps;   // warps per CTA
    const WarpLayout L(B.seg_words, B.lut_entries, B.stage_bytes, NW);
    uint32_t *sym_tab = reinterpret_cast<uint32_t *>(smem);
    uint16_t *mask_tab = reinterpret_cast<uint16_t *>(smem + kFastSize * 4);
    uint8_t *cnt_tab = smem + kFastSize * 6;
    uint16_t *lut = reinterpret_cast<uint16_t *>(smem + kFastBytes);
    uint8_t *buf = smem + L.warp0 + warp * L.warp_bytes;
    const uint32_t *seg = reinterpret_cast<const uint32_t *>(buf);
    const uint8_t *gapb = buf + L.seg_bytes;
    uint8_t *stage = buf + L.stage;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.bars) + warp;
    const uint32_t seg_bytes = L.seg_bytes;
    const uint32_t cbits = B.chunk_words * 32u;

    const uint32_t W = B.total_work, G = gridDim.x;
    const uint32_t w_begin = (uint32_t)((uint64_t)W * blockIdx.x / G);
    const uint32_t w_end = (uint32_t)((uint64_t)W * (blockIdx.x + 1) / G);
    if (w_begin >= w_end) return;
    if (lane == 0) {
        dev::mbar_init(bar, 1);
        dev::fence_mbar_init();
    }
    __syncwarp();

    uint32_t bad = 0, items = 0;
    bool dead = false;   // a bounded wait gave up: this warp stops decoding
    uint32_t ti = locate(B, w_begin, 0);
    for (uint32_t w0 = w_begin; w0 < w_end;) {
        const Df11Tensor &tn = B.t[ti];
        const uint32_t t_end = ti + 1 < B.count ? B.t[ti + 1].first_work : W;
        const uint32_t s_end = min(w_end, t_end);
        // this tensor's tables (every warp is done with the previous ones)
        __syncthreads();
        const uint32_t ntab = min(tn.n_tables, B.lut_entries / 256u);
        for (uint32_t i = tid; i < ntab * 128u; i += blockDim.x)
            reinterpret_cast<uint32_t *>(lut)[i] = reinterpret_cast<const uint32_t *>(tn.lut)[i];
        __syncthreads();
        build_fast_tables(lut, ntab, cnt_tab, mask_tab, sym_tab);
        __syncthreads();

        uint32_t w = w0 + warp;
        if (w < s_end && lane == 0 && !dead) {
            dev::fence_proxy_async_smem();
            issue_warp_item(B, tn, w - tn.first_work, buf, seg_bytes, bar);
        }
        uint64_t o0n = 0, o1n = 0;
        if (w < s_end) {
            o0n = tn.blkoff[w - tn.first_work];
            o1n = tn.blkoff[w - tn.first_work + 1];
        }
        for (; w < s_end && !dead; w += NW) {
            const uint32_t b = w - tn.first_work;
            const uint64_t o0 = o0n, o1 = o1n;
            const bool more = w + NW < s_end;
            if (more) {
                o0n = tn.blkoff[b + NW];
                o1n = tn.blkoff[b + NW + 1];
            }
            const bool ok = o0 <= o1 && o1 <= tn.n && o1 - o0 + 16 <= B.stage_bytes;
            const uint64_t g_lo = (o0 + 15) & ~15ull, g_hi = o1 & ~15ull;
            uint4 sv[kWarpMergeRegs];
#pragma unroll
            for (int m = 0; m < kWarpMergeRegs; m++) {
                const uint64_t g = g_lo + 16ull * (lane + 32u * (uint32_t)m);
                sv[m] = (ok && g < g_hi) ? __ldg(reinterpret_cast<const uint4 *>(tn.sm + g)) : make_uint4(0, 0, 0, 0);
            }
            const bool arrived = dev::mbar_wait_bounded(bar, items & 1u);
            items++;
            if (__any_sync(0xFFFFFFFFu, !arrived)) {
                // let the late copy land (bounded) before this warp stops
                bad |= LWC_DEVICE_TIMEOUT;
                if (lane == 0) dev::mbar_wait_bounded(bar, (items - 1) & 1u);
                dead = true;
                break;
            }
            bool next_issued = false;
            if (ok) {
                const uint64_t rem_block = tn.total_bits - (uint64_t)b * 32u * cbits;
                const uint32_t start = lane * cbits + gapb[lane];
                const bool has_next = lane + 1 < 32u || b + 1 < tn.n_blocks;
                const uint64_t next = has_next ? (uint64_t)(lane + 1) * cbits + gapb[lane + 1] : rem_block;
                const uint32_t end = (uint32_t)min(next, rem_block);

                uint32_t count = 0;
                if (start < end) {
                    uint32_t pos = start, rem = end - start, acc = 0, sbits = 0, scount = 0;
                    Window win(seg, start);
                    for (;;) {
                        const uint32_t wv = win.at(seg, pos);
                        const uint32_t idx = wv >> (32 - kFastBits);
                        const uint32_t e = cnt_tab[idx];
                        const uint32_t len = e & 15u;
                        const uint32_t e2 = cnt_tab[(wv << len) >> (32 - kFastBits)];
                        const uint32_t l2 = e2 & 15u;
                        if ((len - 1u < rem) & (l2 - 1u < rem - len)) {
                            acc += e + e2;
                            pos += len + l2;
                            rem -= len + l2;
                            continue;
                        }
                        if (len - 1u < rem) {
                            acc += e;
                            pos += len;
                            rem -= len;
                            continue;
                        }
                        if (rem == 0) break;
                        if (e == 0) {
                            const uint32_t l = lut_walk(lut, ntab, wv, bad) >> 8;
                            if (l > rem) {
                                bad |= LWC_DEVICE_BAD_CODE;
                                break;
                            }
                            pos += l;
                            rem -= l;
                            sbits += l;
                            scount++;
                            continue;
                        }
                        scount += __popc(mask_tab[idx] & ((1u << rem) - 1u));
                        break;
                    }
                    count = ((acc - (pos - start - sbits)) >> 4) + scount;
                }

                // warp scan of the counts
                uint32_t x = count;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
                    if (lane >= (uint32_t)o) x += y;
                }
                const uint32_t total = __shfl_sync(0xFFFFFFFFu, x, 31);
                const uint32_t first = x - count;
                if (total == (uint32_t)(o1 - o0)) {
                    if (start < end) {
                        uint8_t *bp = stage + (uint32_t)(o0 & 15u) + first;
                        uint32_t pos = start, rem = end - start;
                        Window win(seg, start);
                        for (;;) {
                            const uint32_t wv = win.at(seg, pos);
                            const uint32_t idx = wv >> (32 - kFastBits);
                            const uint32_t e = sym_tab[idx];
                            const uint32_t len = e >> 26;
                            const uint32_t e2 = sym_tab[(wv << len) >> (32 - kFastBits)];
                            const uint32_t l2 = e2 >> 26;
                            if ((len - 1u < rem) & (l2 - 1u < rem - len)) {
                                // n is 1..3: bit 25 set means n >= 2, bits 24 and 25 set mean n = 3
                                const uint32_t n = (e >> 24) & 3u, n2 = (e2 >> 24) & 3u;
                                bp[0] = (uint8_t)e;
                                if (e & (1u << 25)) bp[1] = (uint8_t)(e >> 8);
                                if ((e & 0x3000000u) == 0x3000000u) bp[2] = (uint8_t)(e >> 16);
                                uint8_t *bq = bp + n;
                                bq[0] = (uint8_t)e2;
                                if (e2 & (1u << 25)) bq[1] = (uint8_t)(e2 >> 8);
                                if ((e2 & 0x3000000u) == 0x3000000u) bq[2] = (uint8_t)(e2 >> 16);
                                bp = bq + n2;
                                pos += len + l2;
                                rem -= len + l2;
                                continue;
                            }
                            if (len - 1u < rem) {
                                const uint32_t n = (e >> 24) & 3u;
                                bp[0] = (uint8_t)e;
                                if (n > 1) bp[1] = (uint8_t)(e >> 8);
                                if (n > 2) bp[2] = (uint8_t)(e >> 16);
                                bp += n;
                                pos += len;
                                rem -= len;
                                continue;
                            }
                            if (rem == 0) break;
                            if (e == 0) {
                                const uint32_t r = lut_walk(lut, ntab, wv, bad);
                                const uint32_t l = r >> 8;
                                if (l > rem) break;
                                *bp++ = (uint8_t)r;
                                pos += l;
                                rem -= l;
                                continue;
                            }
                            const uint32_t j = __popc(mask_tab[idx] & ((1u << rem) - 1u));   // < 3
                            if (j > 0) bp[0] = (uint8_t)e;
                            if (j > 1) bp[1] = (uint8_t)(e >> 8);
                            break;
                        }
                    }
                    __syncwarp();
                    // the segment is free: fetch this warp's next block while merging this one
                    if (lane == 0 && more) {
                        dev::fence_proxy_async_smem();
                        issue_warp_item(B, tn, b + NW, buf, seg_bytes, bar);
                    }
                    next_issued = true;

                    if constexpr (LIN) {
                        lin_block<LIN>(*X, ti, tn, stage, sv, o0, o1, g_lo, g_hi, lane);
                    } else {
                        // 32-bit offsets from the block's first 16-weight group
                        const uint64_t base = o0 & ~15ull;
                        const uint32_t rlo = (uint32_t)(g_lo - base), rhi = (uint32_t)(g_hi - base);
                        // typed output and low-mantissa pointers at the block's first group
                        void *ob = E == LWC_ELEM_FP32 ? static_cast<void *>(reinterpret_cast<uint32_t *>(tn.out) + base)
                                                      : static_cast<void *>(tn.out + base);
                        const uint8_t *lb = E == LWC_ELEM_FP32 ? tn.lo + 2 * base : tn.lo;
                        const uint64_t g0 = base / 16;   // first group, for the FP16 tails
                        const uint8_t *sb = tn.sm + base;
    #pragma unroll
                        for (int m = 0; m < kWarpMergeRegs; m++) {
                            const uint32_t r = rlo + 16u * (lane + 32u * (uint32_t)m);
                            if (r < rhi) merge_group<E>(sv[m], *reinterpret_cast<const uint4 *>(stage + r), ob, lb, r, g0);
                        }
                        for (uint32_t r = rlo + 16u * (lane + 32u * (uint32_t)kWarpMergeRegs); r < rhi; r += 512u)
                            merge_group<E>(__ldg(reinterpret_cast<const uint4 *>(sb + r)),
                                           *reinterpret_cast<const uint4 *>(stage + r), ob, lb, r, g0);
                        // partial 16-groups at both ends
                        const uint64_t i = lane < 16 ? o0 + lane : max(g_hi, g_lo) + (lane - 16);
                        const bool head = lane < 16 && i < min(g_lo, o1);
                        const bool tail = lane >= 16 && i < o1;
                        if (head || tail) merge_one<E>(tn.sm[i], stage[i - base], tn.out, tn.lo, i);
                    }
                } else {
                    bad |= LWC_DEVICE_BAD_COUNT;
                }
            } else {
                bad |= LWC_DEVICE_BAD_OFFSET;
            }
            __syncwarp();   // segment and staging area free again
            if (lane == 0 && !next_issued && more) {
                dev::fence_proxy_async_smem();
                issue_warp_item(B, tn, b + NW, buf, seg_bytes, bar);
            }
        }
        w0 = s_end;
        if (w0 < w_end) ti = locate(B, w0, ti);
    }
    if (bad && B.status) atomicOr(B.status, bad);
}

template <int E>
__global__ void __launch_bounds__(kWarpsPerCta * 32, kWarpCtasPerSm) df11_warp_kernel(const __grid_constant__ Df11Batch B) {
    df11_warp_body<E, 0>(B, nullptr);
}

// The counted decoder's body. LIN = 0: merge and store the weights (decoder).
// LIN > 0: dot them with up to LIN activation rows instead (fused linear
// layer, BF16 elements only), as in df11_warp_body.
// FX: the launch's codes have no word longer than 8 bits, and tensors whose
// words all have one length take the fixed-length path (a kernel of its own:
// with FX = 0 the path is compiled out and the variable-length path keeps its
// registers).
template <int E, int LIN, bool FX = false>
__device__ __forceinline__ void df11_counted_body(const Df11Batch &B, const Df11Lin *X) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
    const uint32_t NW = B.warps;
    const CountedLayout L(B.seg_words, B.lut_entries, B.stage_bytes, NW);
    uint2 *sym = reinterpret_cast<uint2 *>(smem);
    uint32_t *sub = reinterpret_cast<uint32_t *>(smem + kFastSize * 8);
    uint16_t *lut = reinterpret_cast<uint16_t *>(smem + kCtdTabBytes);
    uint8_t *buf = smem + L.warp0 + warp * L.warp_bytes;
    const uint32_t *seg = reinterpret_cast<const uint32_t *>(buf);
    const uint8_t *gapb = buf + L.gaps;
    const uint8_t *cntb = buf + L.counts;
    uint32_t *slot = reinterpret_cast<uint32_t *>(buf + L.slot) + lane;
    const uint32_t slot_a = dev::smem_u32(slot), stage_a = dev::smem_u32(buf + L.stage);
    uint8_t *stage = buf + L.stage;
    uint32_t *first_long = reinterpret_cast<uint32_t *>(smem + L.misc);
    uint32_t *claim = first_long + 1;   // the CTA's next unclaimed block of the current tensor
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + L.bars) + warp;
    const uint32_t seg_bytes = L.seg_bytes, last = B.seg_words - 1;
    const uint32_t cbits = B.chunk_words * 32u;

    const uint32_t W = B.total_work, G = gridDim.x;
    const uint32_t w_begin = (uint32_t)((uint64_t)W * blockIdx.x / G);
    const uint32_t w_end = (uint32_t)((uint64_t)W * (blockIdx.x + 1) / G);
    if (w_begin >= w_end) return;
    if (lane == 0) {
        dev::mbar_init(bar, 1);
        dev::fence_mbar_init();
    }
    __syncwarp();

    uint32_t bad = 0, items = 0;
    bool dead = false;   // a bounded wait gave up: this warp stops decoding
    uint32_t ti = locate(B, w_begin, 0);
    for (uint32_t w0 = w_begin; w0 < w_end;) {
        const Df11Tensor &tn = B.t[ti];
        const uint32_t t_end = ti + 1 < B.count ? B.t[ti + 1].first_work : W;
        const uint32_t s_end = min(w_end, t_end);
        __syncthreads();   // every warp is done with the previous tensor's tables and its own buffers
        // warps take the tensor's first blocks in order, then claim one block
        // at a time (so they finish together); the first block's copies
        // overlap the table build
        if (tid == 0) *claim = w0 + NW;
        uint32_t w = w0 + warp;
        uint64_t o0n = 0, o1n = 0;
        if (w < s_end) {
            o0n = tn.blkoff[w - tn.first_work];
            o1n = tn.blkoff[w - tn.first_work + 1];
            if (!dead) issue_counted_item(tn, B.chunk_words, w - tn.first_work, buf, seg_bytes, bar, lane);
        }
        const uint32_t ntab = min(tn.n_tables, B.lut_entries / 256u);
        for (uint32_t i = tid; i < ntab * 128u; i += blockDim.x)
            reinterpret_cast<uint32_t *>(lut)[i] = reinterpret_cast<const uint32_t *>(tn.lut)[i];
        __syncthreads();
        build_counted_tables(lut, ntab, sym, sub, first_long, tid, blockDim.x, [] { __syncthreads(); });
        __syncthreads();
        const uint32_t v0 = *first_long;
        // A code whose words all have one length L <= 8 (then every 11-bit window
        // decodes the same number of codes in the same number of bits, and only
        // then): its codes are fixed-width fields, decoded by direct indexing of a
        // 2^L-entry table (in place of the second-level tables, which such a code
        // does not use)
        if constexpr (FX && !LIN) {
            if (const uint32_t fixed_mode = fixed_code_length(sym, sub, tid, blockDim.x)) {
                const uint32_t fixed_len = fixed_mode & 15u;
                // the copy of this warp's first block, issued before the tables: let it land
                if (w < s_end && !dead) {
                    const bool arrived = dev::mbar_wait_bounded(bar, items & 1u);
                    items++;
                    if (__any_sync(0xFFFFFFFFu, !arrived)) {
                        bad |= LWC_DEVICE_TIMEOUT;
                        if (lane == 0) dev::mbar_wait_bounded(bar, (items - 1) & 1u);
                        dead = true;
                    }
                }
                // this CTA's blocks of the tensor hold weights [ob, oe); adjacent CTAs share
                // their boundary offset, so the ranges tile [0, n) when the tensor's first
                // offset is 0, its last is n and every range is ordered
                const uint32_t b0 = w0 - tn.first_work, b1 = s_end - tn.first_work;
                const uint64_t ob = tn.blkoff[b0], oe = tn.blkoff[b1];
                if (!(ob <= oe && oe <= tn.n && (b0 != 0 || ob == 0) && (b1 != tn.n_blocks || oe == tn.n)))
                    bad |= LWC_DEVICE_BAD_OFFSET;
                else if (tn.total_bits != tn.n * fixed_len)   // L bits per weight, nothing else
                    bad |= LWC_DEVICE_BAD_COUNT;
                else
                    decode_fixed<E>(fixed_mode, tn, sub, ob, oe, tid, blockDim.x);
                w = s_end;   // no block loop
            }
        }

        while (w < s_end && !dead) {
            const uint32_t b = w - tn.first_work;
            const uint64_t o0 = o0n, o1 = o1n;
            uint32_t wn = 0;   // this warp's next block
            if (lane == 0) wn = atomicAdd(claim, 1u);
            wn = __shfl_sync(0xFFFFFFFFu, wn, 0);
            const bool more = wn < s_end;
            if (more) {
                o0n = tn.blkoff[wn - tn.first_work];
                o1n = tn.blkoff[wn - tn.first_work + 1];
            }
            const bool ok = o0 <= o1 && o1 <= tn.n && o1 - o0 + 16 <= B.stage_bytes;
            if (lane == 0 && ok && o1 > o0 && o1 - o0 < (1u << 20))   // this block's sign|mantissa bytes into L2
                dev::prefetch_l2(tn.sm + (o0 & ~15ull), (uint32_t)(((o1 + 15) & ~15ull) - (o0 & ~15ull)));
            // merge units: 16-weight groups, or for BF16 8-weight units (one
            // 16-byte store each, so a warp's store covers 512 contiguous bytes);
            // the sign|mantissa bytes of each lane's first units are loaded now
            constexpr uint32_t U = E == LWC_ELEM_BF16 && !LIN ? 8u : 16u;
            const uint64_t g_lo = (o0 + U - 1) & ~(uint64_t)(U - 1), g_hi = o1 & ~(uint64_t)(U - 1);
            uint4 sv[kWarpMergeRegs];
            // 32-bit offsets from the block's first unit (a block decodes fewer than 2^32 weights)
            const uint32_t span = ok && g_hi > g_lo ? (uint32_t)(g_hi - g_lo) : 0u;
            const uint8_t *smu = tn.sm + g_lo;
#pragma unroll
            for (int m = 0; m < kWarpMergeRegs; m++) {
                if constexpr (U == 8) {
                    const uint32_t g = 8u * (lane + 64u * (uint32_t)m), h = g + 256;
                    const uint2 a = g < span ? __ldg(reinterpret_cast<const uint2 *>(smu + g)) : make_uint2(0, 0);
                    const uint2 c = h < span ? __ldg(reinterpret_cast<const uint2 *>(smu + h)) : make_uint2(0, 0);
                    sv[m] = make_uint4(a.x, a.y, c.x, c.y);
                } else {
                    const uint64_t g = g_lo + 16ull * (lane + 32u * (uint32_t)m);
                    sv[m] = (ok && g < g_hi) ? __ldg(reinterpret_cast<const uint4 *>(tn.sm + g)) : make_uint4(0, 0, 0, 0);
                }
            }
            const bool arrived = dev::mbar_wait_bounded(bar, items & 1u);
            items++;
            if (__any_sync(0xFFFFFFFFu, !arrived)) {
                // let the late copy land (bounded) before this warp stops
                bad |= LWC_DEVICE_TIMEOUT;
                if (lane == 0) dev::mbar_wait_bounded(bar, (items - 1) & 1u);
                dead = true;
                break;
            }
            bool next_issued = false;
            if (ok) {
                // output positions: a warp scan of the stored counts
                const uint32_t cnt = cntb[lane];
                uint32_t x = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
                    if (lane >= (uint32_t)o) x += y;
                }
                const uint32_t total = __shfl_sync(0xFFFFFFFFu, x, 31);
                if (total == (uint32_t)(o1 - o0)) {
                    const uint32_t first = x - cnt;
                    const uint32_t qb = (uint32_t)(o0 & 15u) + first;   // staging byte of this lane's first exponent
                    const uint64_t rem_block = tn.total_bits - (uint64_t)b * 32u * cbits;
                    const uint32_t start = lane * cbits + gapb[lane];
                    const bool has_next = lane + 1 < 32u || b + 1 < tn.n_blocks;
                    const uint64_t next = has_next ? (uint64_t)(lane + 1) * cbits + gapb[lane + 1] : rem_block;
                    const uint32_t end = (uint32_t)min(next, rem_block);
                    if (cnt) {
                        const uint32_t got = decode_counted(seg, last, sym, sub, v0, lut, ntab, start, cnt, qb,
                                                            stage_a, slot_a, bad);
                        // the last step may decode past the lane's codes (by at most 40 bits);
                        // falling short of the next chunk's first code, or far past it, means a bad count
                        if (got - end > 40u) bad |= LWC_DEVICE_BAD_COUNT;
                    }
                    __syncwarp();
                    // the bytes of this lane's first, shared word
                    if ((qb & 3u) && cnt) {
                        const uint32_t hw = *slot, j0 = qb & 3u;
                        uint8_t *hb = stage + (qb & ~3u);
                        hb[j0] = (uint8_t)(hw >> (8 * j0));
                        if (j0 < 3 && cnt > 1) hb[j0 + 1] = (uint8_t)(hw >> (8 * j0 + 8));
                        if (j0 == 1 && cnt > 2) hb[3] = (uint8_t)(hw >> 24);
                    }
                    __syncwarp();
                    // the segment is free: fetch this warp's next block while merging this one
                    if (more) issue_counted_item(tn, B.chunk_words, wn - tn.first_work, buf, seg_bytes, bar, lane);
                    next_issued = true;

                    if constexpr (LIN) {
                        lin_block<LIN, true>(*X, ti, tn, stage, sv, o0, o1, g_lo, g_hi, lane);
                    } else {
                    // 32-bit offsets from the block's first 16-weight group
                    const uint64_t base = o0 & ~15ull;
                    const uint32_t rlo = (uint32_t)(g_lo - base), rhi = (uint32_t)(g_hi - base);
                    const uint8_t *sb = tn.sm + base;
                    if constexpr (E == LWC_ELEM_BF16) {
                        uint16_t *ob = tn.out + base;
                        auto merge8 = [&](uint32_t r, uint32_t sx, uint32_t sy) {
                            const uint2 e = *reinterpret_cast<const uint2 *>(stage + r);
                            uint4 o;
                            merge4r(sx, e.x, o.x, o.y);
                            merge4r(sy, e.y, o.z, o.w);
                            *reinterpret_cast<uint4 *>(ob + r) = o;
                        };
#pragma unroll
                        for (int m = 0; m < kWarpMergeRegs; m++) {
                            const uint32_t r = rlo + 8u * (lane + 64u * (uint32_t)m);
                            if (r < rhi) merge8(r, sv[m].x, sv[m].y);
                            if (r + 256 < rhi) merge8(r + 256, sv[m].z, sv[m].w);
                        }
                        // the rest, loads issued four at a time
                        for (uint32_t r0 = rlo + 8u * (lane + 64u * (uint32_t)kWarpMergeRegs); r0 < rhi; r0 += 1024u) {
                            uint2 q[4];
#pragma unroll
                            for (int j = 0; j < 4; j++) {
                                const uint32_t r = r0 + 256u * j;
                                q[j] = r < rhi ? __ldg(reinterpret_cast<const uint2 *>(sb + r)) : make_uint2(0, 0);
                            }
#pragma unroll
                            for (int j = 0; j < 4; j++)
                                if (r0 + 256u * j < rhi) merge8(r0 + 256u * j, q[j].x, q[j].y);
                        }
                    } else {
                        void *ob = E == LWC_ELEM_FP32 ? static_cast<void *>(reinterpret_cast<uint32_t *>(tn.out) + base)
                                                      : static_cast<void *>(tn.out + base);
                        const uint8_t *lb = E == LWC_ELEM_FP32 ? tn.lo + 2 * base : tn.lo;
                        const uint64_t g0 = base / 16;
#pragma unroll
                        for (int m = 0; m < kWarpMergeRegs; m++) {
                            const uint32_t r = rlo + 16u * (lane + 32u * (uint32_t)m);
                            if (r < rhi) merge_group<E, true>(sv[m], *reinterpret_cast<const uint4 *>(stage + r), ob, lb, r, g0);
                        }
                        for (uint32_t r = rlo + 16u * (lane + 32u * (uint32_t)kWarpMergeRegs); r < rhi; r += 512u)
                            merge_group<E, true>(__ldg(reinterpret_cast<const uint4 *>(sb + r)),
                                           *reinterpret_cast<const uint4 *>(stage + r), ob, lb, r, g0);
                    }
                    // single weights before the first unit (lanes 0-15) and after the last (lanes 16-31)
                    const uint64_t i = lane < 16 ? o0 + lane : max(g_hi, g_lo) + (lane - 16);
                    const bool head = lane < 16 && i < min(g_lo, o1);
                    const bool tail = lane >= 16 && i < o1;
                    if (head || tail) merge_one<E, true>(tn.sm[i], stage[i - base], tn.out, tn.lo, i);
                    }
                } else {
                    bad |= LWC_DEVICE_BAD_COUNT;
                }
            } else {
                bad |= LWC_DEVICE_BAD_OFFSET;
            }
            __syncwarp();   // segment and staging area free again
            if (!next_issued && more) issue_counted_item(tn, B.chunk_words, wn - tn.first_work, buf, seg_bytes, bar, lane);
            w = wn;
        }
        w0 = s_end;
        if (w0 < w_end) ti = locate(B, w0, ti);
    }
    if (bad && B.status) atomicOr(B.status, bad);
}

template <int E, bool FX = false, bool WIDE = false>
__global__ void __launch_bounds__(WIDE ? kWideWarpsPerCta * 32 : kWarpsPerCta * 32, WIDE ? 1 : kWarpCtasPerSm)
    df11_counted_kernel(const __grid_constant__ Df11Batch B) {
    df11_counted_body<E, 0, FX>(B, nullptr);
}

// Fused decode + linear layer on blobs with stored chunk counts (BF16, blocks
// of 32 chunks), for up to MM activation rows.
template <int MM>
__global__ void __launch_bounds__(kWarpsPerCta * 32, MM == 1 ? kWarpCtasPerSm : 1)
    df11_counted_linear_kernel(const __grid_constant__ Df11Batch B, const __grid_constant__ Df11Lin X) {
    df11_counted_body<LWC_ELEM_BF16, MM>(B, &X);
}

// Fused decode + linear layer (BF16 elements, blocks of 32 chunks) for up
// to MM activation rows; with more than one row the accumulators need more
// registers than two CTAs per SM leave.
template <int MM>
__global__ void __launch_bounds__(kWarpsPerCta * 32, MM == 1 ? kWarpCtasPerSm : 1)
    df11_warp_linear_kernel(const __grid_constant__ Df11Batch B, const __grid_constant__ Df11Lin X) {
    df11_warp_body<LWC_ELEM_BF16, MM>(B, &X);
}

using LinKernel = void (*)(Df11Batch, Df11Lin);
const LinKernel kLinKernels[4] = {df11_warp_linear_kernel<1>, df11_warp_linear_kernel<2>, df11_warp_linear_kernel<4>,
                                  df11_warp_linear_kernel<8>};
const LinKernel kCtdLinKernels[4] = {df11_counted_linear_kernel<1>, df11_counted_linear_kernel<2>,
                                     df11_counted_linear_kernel<4>, df11_counted_linear_kernel<8>};
int lin_index(uint32_t M) { return M <= 1 ? 0 : M <= 2 ? 1 : M <= 4 ? 2 : 3; }

// One exponent value for the whole tensor: out = merge(const_exp, sm).
template <int E>
__global__ void df11_const_kernel(const uint8_t *__restrict__ sm, const uint8_t *__restrict__ lo, void *out, uint64_t n,
                                  uint32_t const_exp) {
    const uint32_t e4 = const_exp * 0x01010101u;
    const uint4 ev = make_uint4(e4, e4, e4, e4);
    const uint64_t stride = 16ull * gridDim.x * blockDim.x;
    for (uint64_t g = 16ull * (blockIdx.x * (uint64_t)blockDim.x + threadIdx.x); g < n; g += stride) {
        if (g + 16 <= n) {
            merge_group<E>(__ldg(reinterpret_cast<const uint4 *>(sm + g)), ev, out, lo, g);
        } else {
            for (uint64_t i = g; i < n; i++) merge_one<E>(sm[i], const_exp, out, lo, i);
        }
    }
}

// ---- host side -----------------------------------------------------------------------

struct DeviceConfig {
    int sms = 0;
    int max_smem = 0;
    bool ready = false;
};

std::mutex g_cfg_mutex;
std::vector<DeviceConfig> g_cfg;

lwc_status device_config(DeviceConfig &out) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
    std::lock_guard<std::mutex> lock(g_cfg_mutex);
    if ((int)g_cfg.size() <= dev) g_cfg.resize(dev + 1);
    DeviceConfig &c = g_cfg[dev];
    if (!c.ready) {
        err = cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev);
        if (err == cudaSuccess) err = cudaDeviceGetAttribute(&c.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        const void *kernels[] = {
            (const void *)df11_decode_kernel<256, LWC_ELEM_BF16>, (const void *)df11_decode_kernel<1024, LWC_ELEM_BF16>,
            (const void *)df11_warp_kernel<LWC_ELEM_BF16>,
            (const void *)df11_decode_kernel<256, LWC_ELEM_FP32>, (const void *)df11_decode_kernel<1024, LWC_ELEM_FP32>,
            (const void *)df11_warp_kernel<LWC_ELEM_FP32>,
            (const void *)df11_decode_kernel<256, LWC_ELEM_FP16>, (const void *)df11_decode_kernel<1024, LWC_ELEM_FP16>,
            (const void *)df11_warp_kernel<LWC_ELEM_FP16>, (const void *)df11_counted_kernel<LWC_ELEM_BF16>,
            (const void *)df11_counted_kernel<LWC_ELEM_FP32>, (const void *)df11_counted_kernel<LWC_ELEM_FP16>,
            (const void *)df11_counted_kernel<LWC_ELEM_BF16, true>, (const void *)df11_counted_kernel<LWC_ELEM_FP32, true>,
            (const void *)df11_counted_kernel<LWC_ELEM_FP16, true>,
            (const void *)df11_counted_kernel<LWC_ELEM_BF16, false, true>,
            (const void *)df11_counted_kernel<LWC_ELEM_FP32, false, true>,
            (const void *)df11_counted_kernel<LWC_ELEM_FP16, false, true>,
            (const void *)kLinKernels[0], (const void *)kLinKernels[1],
            (const void *)kLinKernels[2], (const void *)kLinKernels[3], (const void *)kCtdLinKernels[0],
            (const void *)kCtdLinKernels[1], (const void *)kCtdLinKernels[2], (const void *)kCtdLinKernels[3]};
        for (const void *k : kernels) {
            if (err == cudaSuccess) err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, c.max_smem);
            if (err == cudaSuccess)
                err = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        }
        if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "device setup: %s", cudaGetErrorString(err));
        c.ready = true;
    }
    out = c;
    return LWC_OK;
}


// Decode kernels: one CTA per block (blocks of 64+ chunks), one warp per
// block (blocks of 32 chunks), or one warp per block with stored chunk counts
// (kModeCountedShort: codes of at most 8 bits, with the fixed-length path;
// kModeCountedWide: one CTA of 32 warps per SM, for long launches).
enum KernelMode { kModeBlock, kModeWarp, kModeCounted, kModeCountedShort, kModeCountedWide };

template <int E>
const void *df11_kernel(KernelMode mode, uint32_t T) {
    return mode == kModeCounted        ? (const void *)df11_counted_kernel<E>
           : mode == kModeCountedShort ? (const void *)df11_counted_kernel<E, true>
           : mode == kModeCountedWide  ? (const void *)df11_counted_kernel<E, false, true>
           : mode == kModeWarp         ? (const void *)df11_warp_kernel<E>
           : T <= 256           ? (const void *)df11_decode_kernel<256, E>
                                : (const void *)df11_decode_kernel<1024, E>;
}

const void *df11_kernel_for(uint32_t elem, KernelMode mode, uint32_t T) {
    if (elem == LWC_ELEM_FP32) return df11_kernel<LWC_ELEM_FP32>(mode, T);
    if (elem == LWC_ELEM_FP16) return df11_kernel<LWC_ELEM_FP16>(mode, T);
    return df11_kernel<LWC_ELEM_BF16>(mode, T);
}

template <int E>
void launch_df11(KernelMode mode, uint32_t T, unsigned grid, uint32_t threads, size_t smem, cudaStream_t stream,
                 const Df11Batch &B) {
    if (mode == kModeCounted)
        df11_counted_kernel<E><<<grid, threads, smem, stream>>>(B);
    else if (mode == kModeCountedWide)
        df11_counted_kernel<E, false, true><<<grid, threads, smem, stream>>>(B);
    else if (mode == kModeCountedShort)
        df11_counted_kernel<E, true><<<grid, threads, smem, stream>>>(B);
    else if (mode == kModeWarp)
        df11_warp_kernel<E><<<grid, threads, smem, stream>>>(B);
    else if (T <= 256)
        df11_decode_kernel<256, E><<<grid, T, smem, stream>>>(B);
    else
        df11_decode_kernel<1024, E><<<grid, T, smem, stream>>>(B);
}

// Shared memory of a per-warp launch with w warps per CTA.
uint64_t warp_smem(const Df11Batch &B, KernelMode mode, uint32_t w) {
    return mode == kModeCounted || mode == kModeCountedShort || mode == kModeCountedWide
               ? CountedLayout(B.seg_words, B.lut_entries, B.stage_bytes, w).total
                                : WarpLayout(B.seg_words, B.lut_entries, B.stage_bytes, w).total;
}

// Warps per CTA of the per-warp kernels: kWarpsPerCta, or fewer when one
// warp's segment buffer and staging area are large (long chunks).
uint32_t warps_that_fit(const Df11Batch &B, int max_smem, KernelMode mode = kModeWarp) {
    uint32_t w = mode == kModeCountedWide ? kWideWarpsPerCta : kWarpsPerCta;
    while (w > 1 && warp_smem(B, mode, w) > (uint64_t)max_smem) w--;
    return w;
}

// Launch one kernel over up to kMaxBatch tensors sharing (element type,
// chunk_bytes, threads_per_block, stored chunk counts or not).
lwc_status launch_group(const std::vector<int> &idx, const lwc_desc *descs, const void *const *d_ins,
                        uint16_t *const *d_outs, uint32_t *d_status, cudaStream_t stream,
                        const DeviceConfig &cfg) {
    Df11Batch B;
    std::memset(&B, 0, sizeof B);
    const lwc_desc &d0 = descs[idx[0]];
    const uint32_t T = d0.threads_per_block;
    B.chunk_words = d0.chunk_bytes / 4;
    B.seg_words = (uint32_t)round_up((uint64_t)T * B.chunk_words + 2, 4);
    uint64_t work = 0, max_count = 0, max_tables = 0;
    for (size_t j = 0; j < idx.size(); j++) {
        const lwc_desc &d = descs[idx[j]];
        const uint8_t *base = static_cast<const uint8_t *>(d_ins[idx[j]]);
        Df11Tensor &t = B.t[j];
        t.stream = reinterpret_cast<const uint32_t *>(base + d.off_stream);
        t.gaps = base + d.off_gaps;
        t.counts = (d.flags & kFlagChunkCounts) ? base + d.off_counts : nullptr;
        t.blkoff = reinterpret_cast<const uint64_t *>(base + d.off_blkoff);
        t.sm = base + d.off_sm;
        t.lo = d.elem != LWC_ELEM_BF16 ? base + d.off_lo : nullptr;
        t.lut = reinterpret_cast<const uint16_t *>(base + d.off_lut);
        t.out = d_outs[idx[j]];
        t.n = d.n;
        t.total_bits = d.total_bits;
        t.stream_bytes = d.stream_bytes;
        t.n_blocks = (uint32_t)d.n_blocks;
        t.n_tables = d.n_tables;
        t.first_work = (uint32_t)work;
        work += d.n_blocks;
        max_count = std::max<uint64_t>(max_count, d.max_block_count);
        max_tables = std::max<uint64_t>(max_tables, d.n_tables);
    }
    if (work > 0xFFFFFFFFull) return fail(LWC_ERR_UNSUPPORTED, "too many blocks in one launch");
    B.count = (uint32_t)idx.size();
    B.total_work = (uint32_t)work;
    B.stage_bytes = (uint32_t)round_up(max_count + 16, 16);
    B.lut_entries = (uint32_t)(max_tables * 256);
    B.status = d_status;
    uint64_t weights = 0;
    for (const int i : idx) weights += descs[i].n;
    const KernelMode mode = T != 32                           ? kModeBlock
                            : !(d0.flags & kFlagChunkCounts) ? kModeWarp
                            : d0.max_len <= 8                ? kModeCountedShort
                            : weights >= kWideMinWeights     ? kModeCountedWide
                                                             : kModeCounted;
    const bool per_warp = mode != kModeBlock;
    B.warps = per_warp ? warps_that_fit(B, cfg.max_smem, mode) : 0;
    const uint32_t threads = per_warp ? B.warps * 32u : T;
    const uint64_t smem = per_warp ? warp_smem(B, mode, B.warps) : Layout(T, B.seg_words, B.lut_entries, B.stage_bytes).total;
    if (smem > (uint64_t)cfg.max_smem)
        return fail(LWC_ERR_UNSUPPORTED, "decoder needs %llu bytes of shared memory (device allows %d)",
                    (unsigned long long)smem, cfg.max_smem);
    const uint32_t elem = d0.elem;
    const void *kernel = df11_kernel_for(elem, mode, T);
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, (int)threads, (size_t)smem);
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "occupancy: %s", cudaGetErrorString(err));
    if (per_sm < 1) return fail(LWC_ERR_UNSUPPORTED, "decoder does not fit on an SM (%u threads, %llu B smem)",
                                threads, (unsigned long long)smem);
    const uint64_t units = per_warp ? (work + B.warps - 1) / B.warps : work;
    const uint64_t grid = std::min<uint64_t>(units, (uint64_t)per_sm * cfg.sms);
    if (elem == LWC_ELEM_FP32)
        launch_df11<LWC_ELEM_FP32>(mode, T, (unsigned)grid, threads, (size_t)smem, stream, B);
    else if (elem == LWC_ELEM_FP16)
        launch_df11<LWC_ELEM_FP16>(mode, T, (unsigned)grid, threads, (size_t)smem, stream, B);
    else
        launch_df11<LWC_ELEM_BF16>(mode, T, (unsigned)grid, threads, (size_t)smem, stream, B);
    err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
    return LWC_OK;
}

// m' and the shifts of div_cols for divisor d (1 <= d < 2^31): l = ceil(log2 d),
// m' = floor(2^32 (2^l - d) / d) + 1, sh1 = min(l, 1), sh2 = max(l - 1, 0).
void division_magic(uint32_t d, uint32_t &magic, uint32_t &shifts) {
    uint32_t l = 0;
    while ((1ull << l) < d) l++;
    magic = (uint32_t)(((((uint64_t)1 << l) - d) << 32) / d + 1);
    shifts = (l < 1 ? l : 1u) | ((l > 0 ? l - 1 : 0u) << 8);
}

// One fused-linear launch over up to kMaxLinBatch tensors sharing chunk_bytes
// (BF16 elements, blocks of 32 chunks); their outputs are already zeroed.
lwc_status launch_linear_group(const std::vector<int> &idx, const lwc_desc *descs, const void *const *d_blobs,
                               const uint64_t *cols, const uint16_t *const *d_xs, uint32_t M, float *const *d_ys,
                               uint32_t *d_status, cudaStream_t stream, const DeviceConfig &cfg) {
    Df11Batch B;
    Df11Lin X;
    std::memset(&B, 0, sizeof B);
    std::memset(&X, 0, sizeof X);
    const lwc_desc &d0 = descs[idx[0]];
    B.chunk_words = d0.chunk_bytes / 4;
    B.seg_words = (uint32_t)round_up((uint64_t)32 * B.chunk_words + 2, 4);
    uint64_t work = 0, max_count = 0, max_tables = 0;
    for (size_t j = 0; j < idx.size(); j++) {
        const int i = idx[j];
        const lwc_desc &d = descs[i];
        const uint8_t *base = static_cast<const uint8_t *>(d_blobs[i]);
        Df11Tensor &t = B.t[j];
        t.stream = reinterpret_cast<const uint32_t *>(base + d.off_stream);
        t.gaps = base + d.off_gaps;
        t.counts = (d.flags & kFlagChunkCounts) ? base + d.off_counts : nullptr;
        t.blkoff = reinterpret_cast<const uint64_t *>(base + d.off_blkoff);
        t.sm = base + d.off_sm;
        t.lut = reinterpret_cast<const uint16_t *>(base + d.off_lut);
        t.n = d.n;
        t.total_bits = d.total_bits;
        t.stream_bytes = d.stream_bytes;
        t.n_blocks = (uint32_t)d.n_blocks;
        t.n_tables = d.n_tables;
        t.first_work = (uint32_t)work;
        work += d.n_blocks;
        max_count = std::max<uint64_t>(max_count, d.max_block_count);
        max_tables = std::max<uint64_t>(max_tables, d.n_tables);
        X.x[j] = d_xs[i];
        X.y[j] = d_ys[i];
        X.cols[j] = (uint32_t)cols[i];
        X.rows[j] = d.n / cols[i];
        division_magic(X.cols[j], X.magic[j], X.shifts[j]);
    }
    if (work > 0xFFFFFFFFull) return fail(LWC_ERR_UNSUPPORTED, "too many blocks in one launch");
    B.count = (uint32_t)idx.size();
    B.total_work = (uint32_t)work;
    B.stage_bytes = (uint32_t)round_up(max_count + 16, 16);
    B.lut_entries = (uint32_t)(max_tables * 256);
    B.status = d_status;
    X.M = M;
    const KernelMode mode = (d0.flags & kFlagChunkCounts) ? kModeCounted : kModeWarp;
    B.warps = warps_that_fit(B, cfg.max_smem, mode);
    const uint32_t threads = B.warps * 32u;
    const uint64_t smem = warp_smem(B, mode, B.warps);
    if (smem > (uint64_t)cfg.max_smem)
        return fail(LWC_ERR_UNSUPPORTED, "decoder needs %llu bytes of shared memory (device allows %d)",
                    (unsigned long long)smem, cfg.max_smem);
    const LinKernel kernel = mode == kModeCounted ? kCtdLinKernels[lin_index(M)] : kLinKernels[lin_index(M)];
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void *)kernel, (int)threads,
                                                                    (size_t)smem);
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "occupancy: %s", cudaGetErrorString(err));
    if (per_sm < 1) return fail(LWC_ERR_UNSUPPORTED, "linear kernel does not fit on an SM");
    const uint64_t grid = std::min<uint64_t>((work + B.warps - 1) / B.warps, (uint64_t)per_sm * cfg.sms);
    kernel<<<(unsigned)grid, threads, (size_t)smem, stream>>>(B, X);
    err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "linear launch: %s", cudaGetErrorString(err));
    return LWC_OK;
}

lwc_status launch_const(const lwc_desc &d, const void *d_in, uint16_t *d_out, cudaStream_t stream,
                        const DeviceConfig &cfg) {
    if (d.n == 0) return LWC_OK;
    const uint64_t groups = (d.n + 15) / 16;
    const uint64_t blocks = std::min<uint64_t>((groups + 255) / 256, (uint64_t)cfg.sms * 8);
    const uint8_t *sm = static_cast<const uint8_t *>(d_in) + d.off_sm;
    const uint8_t *lo = d.elem != LWC_ELEM_BF16 ? static_cast<const uint8_t *>(d_in) + d.off_lo : nullptr;
    if (d.elem == LWC_ELEM_FP32)
        df11_const_kernel<LWC_ELEM_FP32><<<(unsigned)blocks, 256, 0, stream>>>(sm, lo, d_out, d.n, d.const_exp);
    else if (d.elem == LWC_ELEM_FP16)
        df11_const_kernel<LWC_ELEM_FP16><<<(unsigned)blocks, 256, 0, stream>>>(sm, lo, d_out, d.n, d.const_exp);
    else
        df11_const_kernel<LWC_ELEM_BF16><<<(unsigned)blocks, 256, 0, stream>>>(sm, lo, d_out, d.n, d.const_exp);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "decode launch: %s", cudaGetErrorString(err));
    return LWC_OK;
}

}  // namespace
}  // namespace lwc

using namespace lwc;

extern "C" {

lwc_status lwc_decode_dfloat11_batched(const lwc_desc *descs, const void *const *d_ins, uint16_t *const *d_outs,
                                       int count, uint32_t *d_status, lwc_stream_t stream) {
    if (count < 0 || (count > 0 && (!descs || !d_ins || !d_outs)))
        return fail(LWC_ERR_INVALID_ARG, "bad batch arguments");
    for (int i = 0; i < count; i++) {
        lwc_status st = check_df11_desc(&descs[i]);
        if (st) return st;
        if (descs[i].n == 0) continue;
        if (!d_ins[i] || !d_outs[i]) return fail(LWC_ERR_INVALID_ARG, "NULL device pointer (tensor %d)", i);
        if (!aligned16(d_ins[i]) || !aligned16(d_outs[i]))
            return fail(LWC_ERR_MISALIGNED, "device pointers must be 16-byte aligned (tensor %d)", i);
    }
    if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u))
        return fail(LWC_ERR_MISALIGNED, "status word must be 4-byte aligned");
    bool any = false;
    for (int i = 0; i < count; i++) any = any || descs[i].n > 0;
    if (!any) {
        clear_error();
        return LWC_OK;
    }
    DeviceConfig cfg;
    lwc_status st = device_config(cfg);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // single-exponent tensors; the rest grouped by (element type, chunk_bytes, threads_per_block)
    std::vector<std::pair<uint64_t, int>> keyed;
    for (int i = 0; i < count; i++) {
        const lwc_desc &d = descs[i];
        if (d.n == 0) continue;
        if (d.flags & kFlagSingleExponent) {
            st = launch_const(d, d_ins[i], d_outs[i], s, cfg);
            if (st) return st;
            continue;
        }
        const uint64_t counted = (d.flags & kFlagChunkCounts) ? 1 : 0;
        const uint64_t short_codes = counted && d.max_len <= 8 ? 1 : 0;   // the kernel with the fixed-length path
        keyed.push_back({(short_codes << 51) | (counted << 50) | ((uint64_t)d.elem << 40) | ((uint64_t)d.chunk_bytes << 20) |
                             d.threads_per_block,
                         i});
    }
    std::stable_sort(keyed.begin(), keyed.end(),
                     [](const std::pair<uint64_t, int> &a, const std::pair<uint64_t, int> &b) { return a.first < b.first; });
    std::vector<int> group;
    for (size_t i = 0; i < keyed.size(); i++) {
        group.push_back(keyed[i].second);
        const bool last = i + 1 == keyed.size() || keyed[i + 1].first != keyed[i].first;
        if (last || group.size() == (size_t)kMaxBatch) {
            st = launch_group(group, descs, d_ins, d_outs, d_status, s, cfg);
            if (st) return st;
            group.clear();
        }
    }
    clear_error();
    return LWC_OK;
}

lwc_status lwc_decode_dfloat11_checked(const lwc_desc *desc, const void *d_in, uint16_t *d_out, uint32_t *d_status,
                                       lwc_stream_t stream) {
    if (!desc) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    return lwc_decode_dfloat11_batched(desc, &d_in, &d_out, 1, d_status, stream);
}

lwc_status lwc_decode_dfloat11(const lwc_desc *desc, const void *d_in, uint16_t *d_out, lwc_stream_t stream) {
    return lwc_decode_dfloat11_checked(desc, d_in, d_out, nullptr, stream);
}

lwc_status lwc_linear_dfloat11_batched(const lwc_desc *descs, const void *const *d_blobs, const uint64_t *cols,
                                       const uint16_t *const *d_xs, int M, float *const *d_ys, int count,
                                       uint32_t *d_status, lwc_stream_t stream) {
    if (count < 0 || (count > 0 && (!descs || !d_blobs || !cols || !d_xs || !d_ys)))
        return fail(LWC_ERR_INVALID_ARG, "bad batch arguments");
    if (M < 1 || M > kMaxRows) return fail(LWC_ERR_INVALID_ARG, "M must be 1..%d (got %d)", kMaxRows, M);
    bool any = false;
    for (int i = 0; i < count; i++) {
        const lwc_desc &d = descs[i];
        lwc_status st = check_df11_desc(&d);
        if (st) return st;
        if (cols[i] == 0 || cols[i] >= (1ull << 31) || d.n % cols[i] != 0)
            return fail(LWC_ERR_INVALID_ARG, "cols must be 1..2^31-1 and divide n (tensor %d)", i);
        if (d.n == 0) continue;
        any = true;
        if (d.elem != LWC_ELEM_BF16)
            return fail(LWC_ERR_UNSUPPORTED, "the fused linear layer takes BF16 weights (tensor %d)", i);
        if (!(d.flags & kFlagSingleExponent) && d.threads_per_block != 32)
            return fail(LWC_ERR_UNSUPPORTED, "the fused linear layer needs blocks of 32 chunks (tensor %d has %u)", i,
                        d.threads_per_block);
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
    DeviceConfig cfg;
    lwc_status st = device_config(cfg);
    if (st) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::vector<std::pair<uint64_t, int>> keyed;
    for (int i = 0; i < count; i++) {
        const lwc_desc &d = descs[i];
        if (d.n == 0) continue;
        const uint64_t rows = d.n / cols[i];
        if (d.flags & kFlagSingleExponent) {
            const uint64_t blocks = std::min<uint64_t>((rows + 7) / 8, (uint64_t)cfg.sms * 8);
            df11_linear_const_kernel<<<(unsigned)blocks, 256, 0, s>>>(
                static_cast<const uint8_t *>(d_blobs[i]) + d.off_sm, d.const_exp, d_xs[i], (uint32_t)M, rows,
                (uint32_t)cols[i], d_ys[i]);
        } else {
            const uint64_t ny = rows * (uint64_t)M;
            const uint64_t blocks = std::min<uint64_t>((ny + 255) / 256, (uint64_t)cfg.sms * 8);
            zero_f32_kernel<<<(unsigned)blocks, 256, 0, s>>>(d_ys[i], ny);
            keyed.push_back({((uint64_t)((d.flags & kFlagChunkCounts) ? 1 : 0) << 40) | d.chunk_bytes, i});
        }
        cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return fail(LWC_ERR_CUDA, "linear launch: %s", cudaGetErrorString(err));
    }
    std::stable_sort(keyed.begin(), keyed.end(),
                     [](const std::pair<uint64_t, int> &a, const std::pair<uint64_t, int> &b) { return a.first < b.first; });
    std::vector<int> group;
    for (size_t i = 0; i < keyed.size(); i++) {
        group.push_back(keyed[i].second);
        const bool last = i + 1 == keyed.size() || keyed[i + 1].first != keyed[i].first;
        if (last || group.size() == (size_t)kMaxLinBatch) {
            st = launch_linear_group(group, descs, d_blobs, cols, d_xs, (uint32_t)M, d_ys, d_status, s, cfg);
            if (st) return st;
            group.clear();
        }
    }
    clear_error();
    return LWC_OK;
}

lwc_status lwc_linear_dfloat11(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x, int M,
                               float *d_y, uint32_t *d_status, lwc_stream_t stream) {
    if (!desc) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    return lwc_linear_dfloat11_batched(desc, &d_blob, &cols, &d_x, M, &d_y, 1, d_status, stream);
}

}  // extern "C"
