// Device code shared by the DFloat11 kernels (the decoders of lwc_df11.cu
// and the tensor-core matrix product of lwc_gemm.cu): one tensor's device
// view, the walk of the blob's hierarchical lookup tables, the BF16 merge of
// rotated exponents and the counted decoder's pieces (its symbol tables, the
// bulk copies of one block and the decode of one lane's codes into a
// shared-memory staging area).
//
// What they compute ("Koniec z kompromisami! DFloat11 ratuje dokładność
// modeli AI ...", section "Jak to działa w praktyce? Magia na poziomie
// GPU"): each code of the Huffman-coded exponent stream is resolved with
// lookup tables kept in shared memory, and every weight is rebuilt from its
// exponent and its raw sign|mantissa byte.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "lwc_device.cuh"
#include "lwc_internal.h"

namespace lwc {
namespace df11dev {

constexpr int kFastBits = 11;
constexpr int kFastSize = 1 << kFastBits;

struct Df11Tensor {
    const uint32_t *stream;
    const uint8_t *gaps;
    const uint8_t *counts; // per-chunk code counts (blobs that store them), else null
    const uint64_t *blkoff;
    const uint8_t *sm;
    const uint8_t *lo;     // raw low-mantissa section (FP32, FP16 elements)
    const uint16_t *lut;
    uint16_t *out;
    uint64_t n;
    uint64_t total_bits;
    uint64_t stream_bytes;
    uint32_t n_blocks;
    uint32_t n_tables;
    uint32_t first_work;   // index of this tensor's block 0 in the launch's work list
    uint32_t pad;
};

// Walk the hierarchical tables with the 32 stream bits at the current
// position (MSB first); returns symbol | length << 8. A path no valid code
// takes yields length 1 and sets LWC_DEVICE_BAD_CODE in `bad` (so decoding
// always advances and ends).
__device__ __forceinline__ uint32_t lut_walk(const uint16_t *lut, uint32_t ntab, uint32_t w, uint32_t &bad) {
    uint32_t e = lut[w >> 24];
#pragma unroll 1
    for (int d = 1; (e & 0x8000u) && d < 4; d++) {
        const uint32_t t = e & 0x7FFFu;
        if (t >= ntab) {
            bad |= LWC_DEVICE_BAD_CODE;
            return 0x100u;
        }
        e = lut[t * 256u + ((w >> (24 - 8 * d)) & 0xFFu)];
    }
    const uint32_t len = (e >> 8) & 0x3Fu;
    if ((e & 0x8000u) || len == 0 || len > 32) {
        bad |= LWC_DEVICE_BAD_CODE;
        return 0x100u;
    }
    return e & 0x3FFFu;
}

// The same from rotated exponents r = (e >> 1) | (e & 1) << 7, as the counted
// decoder stages them: each byte is then one bit-select of s and r
// (low byte: s's mantissa bits under r's top bit; high byte: r's low seven
// bits under s's sign bit).
__device__ __forceinline__ void merge4r(uint32_t s, uint32_t r, uint32_t &w01, uint32_t &w23) {
    const uint32_t lo = (s & 0x7F7F7F7Fu) | (r & 0x80808080u);
    const uint32_t hi = (r & 0x7F7F7F7Fu) | (s & 0x80808080u);
    w01 = __byte_perm(lo, hi, 0x5140u);
    w23 = __byte_perm(lo, hi, 0x7362u);
}

// The exponent in the low byte of e (higher bits ignored), rotated right by one bit.
__device__ __forceinline__ uint32_t rot_exponent(uint32_t e) {
    e &= 0xFFu;
    return ((e >> 1) | (e << 7)) & 0xFFu;
}

// ---- per-warp blocks with stored chunk counts ------------------------------------
//
// Blobs that store each chunk's code count (flags bit 1) carry the result of
// the first phase of the two-phase decoder: a warp reads the 32 counts of
// its block, turns them into output positions with a warp scan and decodes
// each chunk once. Each lane assembles its exponents into 32-bit words in
// registers and writes whole words to the staging area (a quarter of the
// shared-memory stores of byte writes, and far fewer bank conflicts). The
// word a lane shares with the lane before it (when its first exponent is not
// word aligned) goes to a private slot instead; after the warp's word stores
// the lane copies its bytes of that word into place, so no byte is written
// by two lanes at once. Codes of 12 to 19 bits take one more lookup, in a
// second-level table indexed by the next 8 bits (for the first kSubTables
// 11-bit prefixes that begin long codes: in a canonical code those are the
// numerically last prefixes); longer codes walk the blob's hierarchical
// tables.
//
// Symbol table entry (64 bits, indexed by the next 11 stream bits): the low
// word holds up to four exponents (first code in the low byte, zero bytes
// above them); the high word holds the bits their codes take (bits 0-4) and
// 8 x how many there are (bits 8-13). An all-zero entry means the first code
// is longer than 11 bits. Second-level entries are 32-bit: exponent | 1 <<
// 24 | code length << 27, or 0.

constexpr uint32_t kSubTables = 2;
constexpr uint32_t kCtdTabBytes = kFastSize * 8 + kSubTables * 256 * 4;   // 18 KB

struct CountedLayout {
    uint32_t warp0, seg_bytes, gaps, counts, slot, stage, warp_bytes, misc, bars, total;
    __host__ __device__ CountedLayout(uint32_t seg_words, uint32_t lut_entries, uint32_t stage_bytes, uint32_t warps) {
        warp0 = kCtdTabBytes + ((2 * lut_entries + 15) & ~15u);
        seg_bytes = 4 * seg_words;
        gaps = seg_bytes;     // 48 bytes: the block's 32 gaps, then the next block's first 16
        counts = gaps + 48;   // the block's 32 code counts
        slot = counts + 32;   // one word per lane: its first (shared) staging word
        stage = slot + 128;
        warp_bytes = stage + stage_bytes;
        misc = warp0 + warps * warp_bytes;   // the first long 11-bit prefix; the next unclaimed block
        bars = misc + 16;
        total = bars + 8 * warps;
    }
};

// Symbol table and second-level tables of one tensor, from its hierarchical
// tables: threads t = 0 .. nt - 1 of the CTA take part, and sync() is the
// barrier among them (called twice inside).
template <typename Sync>
__device__ void build_counted_tables(const uint16_t *lut, uint32_t ntab, uint2 *sym, uint32_t *sub,
                                     uint32_t *first_long, uint32_t t, uint32_t nt, Sync sync) {
    if (t == 0) *first_long = kFastSize;
    sync();
    for (uint32_t v = t; v < kFastSize; v += nt) {
        uint32_t w = v << (32 - kFastBits), used = 0, cnt = 0, syms = 0, ignore = 0;
        while (cnt < 4) {
            const uint32_t r = lut_walk(lut, ntab, w, ignore);
            const uint32_t len = r >> 8;
            if (ignore || used + len > (uint32_t)kFastBits) break;
            syms |= rot_exponent(r) << (8 * cnt);
            cnt++;
            used += len;
            w <<= len;
        }
        sym[v] = cnt ? make_uint2(syms, used | (cnt << 11)) : make_uint2(0u, 0u);
        if (!cnt) atomicMin(first_long, v);
    }
    sync();
    const uint32_t v0 = *first_long;
    for (uint32_t i = t; i < kSubTables * 256u; i += nt) {
        const uint32_t v = v0 + (i >> 8);
        uint32_t e = 0;
        if (v < (uint32_t)kFastSize) {
            uint32_t ignore = 0;
            const uint32_t r = lut_walk(lut, ntab, (v << (32 - kFastBits)) | ((i & 255u) << (24 - kFastBits)), ignore);
            const uint32_t len = r >> 8;
            if (!ignore && len > (uint32_t)kFastBits && len <= (uint32_t)kFastBits + 8) e = rot_exponent(r) | (1u << 24) | (len << 27);
        }
        sub[i] = e;
    }
}

// Lanes 0-2 of a warp (all lanes call it): the bulk copies of block b of
// tensor `tn` into the warp's buffer -- lane 0 its stream segment, lane 1 its
// 32 gaps (+ the next block's first 16), lane 2 its 32 code counts -- on one
// mbarrier, whose transaction count lane 0 sets first.
__device__ __forceinline__ void issue_counted_item(const Df11Tensor &tn, uint32_t chunk_words, uint32_t b, uint8_t *buf,
                                                   uint32_t seg_bytes, uint64_t *bar, uint32_t lane) {
    const uint64_t seg0 = (uint64_t)b * 32u * chunk_words * 4;   // multiple of 128
    const uint64_t avail = tn.stream_bytes > seg0 ? tn.stream_bytes - seg0 : 0;
    const uint32_t bytes = (uint32_t)(avail < seg_bytes ? avail : seg_bytes);
    const uint32_t gbytes = b + 1 < tn.n_blocks ? 48u : 32u;
    if (lane == 0) {
        dev::fence_proxy_async_smem();   // this warp's reads of the buffer come before the copies' writes
        dev::mbar_arrive_expect_tx(bar, bytes + gbytes + 32u);
    }
    __syncwarp();
    const uint8_t *src = lane == 0 ? reinterpret_cast<const uint8_t *>(tn.stream) + seg0
                         : lane == 1 ? tn.gaps + (uint64_t)b * 32u : tn.counts + (uint64_t)b * 32u;
    const uint32_t n = lane == 0 ? bytes : lane == 1 ? gbytes : 32u;
    if (lane < 3 && n) dev::bulk_g2s(buf + (lane == 0 ? 0u : lane == 1 ? seg_bytes : seg_bytes + 48), src, n, bar);
}

// The 32 stream bits at bit `pos` of the segment, as Window, with the word
// index kept inside the segment buffer whatever the counts say.
struct SegWindow {
    uint32_t wi, w0, w1;
    __device__ __forceinline__ SegWindow(const uint32_t *seg, uint32_t pos, uint32_t last)
        : wi((pos >> 5) - 1u), w0(0), w1(seg[min(pos >> 5, last)]) {}
    __device__ __forceinline__ uint32_t at(const uint32_t *seg, uint32_t pos, uint32_t last) {
        const uint32_t ni = pos >> 5;
        w0 = ni != wi ? w1 : w0;
        w1 = seg[min(ni + 1, last)];
        wi = ni;
        return __funnelshift_l(w1, w0, pos);
    }
};

// Stores v at shared-memory address a when p is non-zero, as a predicated
// instruction (the lanes of a warp take different store paths every step;
// predication keeps them on one instruction stream).
__device__ __forceinline__ void st_shared_if(uint32_t a, uint32_t v, uint32_t p) {
    asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q st.shared.u32 [%0], %1;\n\t}" ::"r"(a), "r"(v),
                 "r"(p)
                 : "memory");
}

// Decodes `cnt` codes from bit `pos` of the segment; exponent j goes to
// staging byte qb + j (stage = the staging area's shared-memory address).
// Words of the staging area that hold none of these exponents are never
// written; the word holding byte qb goes to the lane's slot (shared address
// `slot`) when qb is not word aligned. Each step reads 64 stream bits and
// takes three table entries (up to twelve codes). Returns the bit where
// decoding stopped: the last step takes whole table entries, so that is the
// end of the last code or up to 40 bits past it.
__device__ __forceinline__ uint32_t decode_counted(const uint32_t *seg, uint32_t last, const uint2 *sym,
                                                   const uint32_t *sub, uint32_t v0, const uint16_t *lut,
                                                   uint32_t ntab, uint32_t pos, uint32_t cnt, uint32_t qb,
                                                   uint32_t stage, uint32_t slot, uint32_t &bad) {
    uint32_t nxt = stage + 4 * ((qb >> 2) + 1);     // the staging word after the current one
    uint32_t dst = (qb & 3u) ? slot : nxt - 4;      // where the current word goes
    const uint32_t lim = stage + 4 * ((qb + cnt + 3) >> 2);   // first word past this lane's bytes
    uint32_t lo = 0, sh = (qb & 3u) << 3;           // pending bytes of the current word, and their bits
    int32_t k8 = (int32_t)(cnt << 3);               // exponents still to decode, x 8
    // Appends the n8/8 (<= 4) exponents c (low bytes, zero above them) at
    // byte sh/8 of the current word and stores the word if it is complete and
    // holds one of this lane's exponents (always true when `first`: the
    // step's first entry starts at one of them).
    auto emit = [&](uint32_t c, uint32_t n8, bool first) {
        const uint32_t w = lo | (c << sh);
        const uint32_t spill = __funnelshift_lc(c, 0u, sh);
        sh += n8;
        const uint32_t a = sh >= 32;
        st_shared_if(dst, w, a & (first || nxt - 4 < lim));
        dst = a ? nxt : dst;
        nxt += a << 2;
        lo = a ? spill : w;
        sh &= 31u;
    };
    while (k8 > 0) {
        const uint32_t ni = min(pos >> 5, last - 2);
        const uint32_t hi = __funnelshift_l(seg[ni + 1], seg[ni], pos);       // stream bits pos .. pos + 31
        const uint32_t lw = __funnelshift_l(seg[ni + 2], seg[ni + 1], pos);   // pos + 32 .. pos + 63
        uint2 e1 = sym[hi >> (32 - kFastBits)];
        if (e1.y == 0u) {   // the first code is longer than 11 bits
            const uint32_t s = (hi >> (32 - kFastBits)) - v0;
            const uint32_t r = s < kSubTables ? sub[(s << 8) | ((hi >> (24 - kFastBits)) & 0xFFu)] : 0u;
            if (r == 0u) {   // longer than 19 bits (or a prefix without a second-level table)
                const uint32_t t = lut_walk(lut, ntab, hi, bad);
                emit(rot_exponent(t), 8u, true);
                pos += t >> 8;
                k8 -= 8;
                continue;
            }
            e1 = make_uint2(r & 0xFFu, (r >> 27) | (8u << 8));
        }
        const uint32_t l1 = e1.y & 31u;   // <= 19
        const uint32_t x2 = __funnelshift_l(lw, hi, l1);   // stream bits pos + l1 .. pos + l1 + 31
        const uint2 e2 = sym[x2 >> (32 - kFastBits)];
        const uint32_t l2 = e2.y & 31u;   // <= 11 (0 if the code is long: e3 then reads the same bits)
        const uint2 e3 = sym[(x2 << l2) >> (32 - kFastBits)];
        const uint32_t n1 = e1.y >> 8, n2 = e2.y >> 8, n3 = e3.y >> 8;
        emit(e1.x, n1, true);
        emit(e2.x, n2, false);
        emit(e3.x, n3, false);
        pos += l1 + l2 + (e3.y & 31u);
        k8 -= (int32_t)(n1 + n2 + n3);
    }
    st_shared_if(dst, lo, nxt - 4 < lim);   // the last, partial word
    return pos;
}

// Whole CTA (threads t = 0 .. nt - 1 are all of it), after the symbol table
// is built: L (1..8) when every symbol-table entry holds the same number c of
// codes in the same c L bits with L <= 8, plus kFixedAffine when code word v
// stands for exponent e0 + v for every v; else 0. Equal entries hold exactly
// when every code word has length L: a window that starts with copies of a
// code word of length l decodes min(4, 11 / l) of them in l times as many
// bits, so equal entries give every word the same length, and a word longer
// than 11 bits leaves its windows' entries empty. For such a code, tab[v]
// (v < 2^L, in the second-level tables' place) becomes the rotated exponent
// of code word v.
constexpr uint32_t kFixedAffine = 16;

__device__ __forceinline__ uint32_t fixed_code_length(const uint2 *sym, uint32_t *tab, uint32_t t, uint32_t nt) {
    const uint32_t y0 = sym[0].y, c = y0 >> 11, used = y0 & 31u;
    int same = y0 != 0u;
    for (uint32_t v = t; v < (uint32_t)kFastSize; v += nt) same &= sym[v].y == y0;
    const uint32_t L = c != 0 && used % c == 0 && used / c <= 8 ? used / c : 0u;
    if (!__syncthreads_and(same) || L == 0) return 0;
    for (uint32_t v = t; v < (1u << L); v += nt) tab[v] = sym[v << (kFastBits - L)].x & 0xFFu;
    __syncthreads();
    // the exponent of word v, un-rotated, against that of word 0 plus v
    const uint32_t e0 = ((tab[0] << 1) | (tab[0] >> 7)) & 0xFFu;
    int affine = e0 + (1u << L) - 1u <= 255u;
    for (uint32_t v = t; v < (1u << L); v += nt) affine &= (((tab[v] << 1) | (tab[v] >> 7)) & 0xFFu) == e0 + v;
    return __syncthreads_and(affine) ? L | kFixedAffine : L;
}

}  // namespace df11dev
}  // namespace lwc
