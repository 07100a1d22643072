// Host side of liblwc: the two encoders, the blob header, descriptor checks
// and error reporting.
//
// DFloat11-style encoder: "Koniec z kompromisami! DFloat11 ratuje dokładność
// modeli AI ..." (gadzety360.pl), section "Przełom: DFloat11 – bezstratna
// kompresja z wydajnością GPU" — split BF16 into sign, exponent and mantissa,
// Huffman code the exponent only, keep sign and mantissa as they are. Section
// "Jak to działa w praktyce? Magia na poziomie GPU" motivates what the encoder
// adds for the GPU: small linked lookup tables, and per-chunk / per-block
// start offsets so that the two-phase decoder can start every thread at once.
//
// Codebook encoder: "Codebook Lossless Compression: когда 25% памяти значат
// больше, чем кажется" (ai-manual.ru), section "Как работает эта магия?", and
// "無損 LLM 壓縮減少 10-25% RAM" (setupai.cc), key points — a table of the
// distinct values plus bit-packed indices into it.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "lwc_internal.h"

namespace lwc {

static thread_local std::string g_last_error;

lwc_status fail(lwc_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

void clear_error() { g_last_error.clear(); }

namespace {
template <typename T>
void put(uint8_t *h, size_t off, T v) { std::memcpy(h + off, &v, sizeof v); }
template <typename T>
T get(const uint8_t *h, size_t off) { T v; std::memcpy(&v, h + off, sizeof v); return v; }
}  // namespace

// ---------------------------------------------------------------- header I/O

void write_header(uint8_t *h, const lwc_desc &d) {
    std::memset(h, 0, kHeaderBytes);
    put<uint32_t>(h, 0, d.magic);
    put<uint16_t>(h, 4, (uint16_t)d.version);
    put<uint16_t>(h, 6, (uint16_t)d.codec);
    put<uint64_t>(h, 8, d.n);
    put<uint64_t>(h, 16, d.total_bytes);
    put<uint32_t>(h, 24, kHeaderBytes);
    put<uint32_t>(h, 28, d.flags);
    if (d.codec == LWC_CODEC_DFLOAT11) {
        put<uint32_t>(h, 32, d.chunk_bytes);
        put<uint32_t>(h, 36, d.threads_per_block);
        put<uint32_t>(h, 40, d.max_len);
        put<uint32_t>(h, 44, d.n_tables);
        put<uint64_t>(h, 48, d.n_chunks);
        put<uint64_t>(h, 56, d.n_blocks);
        put<uint64_t>(h, 64, d.total_bits);
        put<uint32_t>(h, 72, d.max_block_count);
        put<uint32_t>(h, 76, d.const_exp);
        put<uint64_t>(h, 80, d.off_lengths);
        put<uint64_t>(h, 88, d.off_lut);
        put<uint64_t>(h, 96, d.off_gaps);
        put<uint64_t>(h, 104, d.off_blkoff);
        put<uint64_t>(h, 112, d.off_stream);
        put<uint64_t>(h, 120, d.stream_bytes);
        put<uint64_t>(h, 128, d.off_sm);
        put<uint32_t>(h, 136, d.elem);
        put<uint64_t>(h, 144, d.off_lo);
        put<uint64_t>(h, 152, d.lo_bytes);
        put<uint64_t>(h, 160, d.off_counts);
    } else {
        put<uint32_t>(h, 32, d.U);
        put<uint32_t>(h, 36, d.k);
        put<uint64_t>(h, 40, d.off_table);
        put<uint64_t>(h, 48, d.off_packed);
        put<uint64_t>(h, 56, d.packed_bytes);
    }
}

namespace {

void read_header(const uint8_t *h, lwc_desc &d) {
    std::memset(&d, 0, sizeof d);
    d.magic = get<uint32_t>(h, 0);
    d.version = get<uint16_t>(h, 4);
    d.codec = get<uint16_t>(h, 6);
    d.n = get<uint64_t>(h, 8);
    d.total_bytes = get<uint64_t>(h, 16);
    d.flags = get<uint32_t>(h, 28);
    if (d.codec == LWC_CODEC_DFLOAT11) {
        d.chunk_bytes = get<uint32_t>(h, 32);
        d.threads_per_block = get<uint32_t>(h, 36);
        d.max_len = get<uint32_t>(h, 40);
        d.n_tables = get<uint32_t>(h, 44);
        d.n_chunks = get<uint64_t>(h, 48);
        d.n_blocks = get<uint64_t>(h, 56);
        d.total_bits = get<uint64_t>(h, 64);
        d.max_block_count = get<uint32_t>(h, 72);
        d.const_exp = get<uint32_t>(h, 76);
        d.off_lengths = get<uint64_t>(h, 80);
        d.off_lut = get<uint64_t>(h, 88);
        d.off_gaps = get<uint64_t>(h, 96);
        d.off_blkoff = get<uint64_t>(h, 104);
        d.off_stream = get<uint64_t>(h, 112);
        d.stream_bytes = get<uint64_t>(h, 120);
        d.off_sm = get<uint64_t>(h, 128);
        d.elem = get<uint32_t>(h, 136);
        d.off_lo = get<uint64_t>(h, 144);
        d.lo_bytes = get<uint64_t>(h, 152);
        d.off_counts = get<uint64_t>(h, 160);
    } else if (d.codec == LWC_CODEC_CODEBOOK) {
        d.U = get<uint32_t>(h, 32);
        d.k = get<uint32_t>(h, 36);
        d.off_table = get<uint64_t>(h, 40);
        d.off_packed = get<uint64_t>(h, 48);
        d.packed_bytes = get<uint64_t>(h, 56);
    }
}

}  // namespace

namespace {

// ------------------------------------------------------------ Huffman code

// Code lengths by the two-queue construction: leaves sorted by count in one
// queue, merged nodes (created in non-decreasing weight) in a second; every
// step merges the two lightest fronts.
void huffman_lengths(const uint64_t counts[256], uint32_t len[256]) {
    std::vector<std::pair<uint64_t, int>> leaves;
    for (int s = 0; s < 256; s++)
        if (counts[s]) leaves.push_back({counts[s], s});
    std::memset(len, 0, 256 * sizeof(uint32_t));
    const int m = (int)leaves.size();
    if (m < 2) return;
    std::sort(leaves.begin(), leaves.end());
    // node ids: 0..m-1 leaves (in sorted order), m.. merged nodes
    std::vector<uint64_t> weight(2 * m - 1);
    std::vector<int> parent(2 * m - 1, -1);
    for (int i = 0; i < m; i++) weight[i] = leaves[i].first;
    int li = 0, mi = m, next = m;
    auto pick = [&]() {
        if (li < m && (mi >= next || weight[li] <= weight[mi])) return li++;
        return mi++;
    };
    for (int step = 0; step < m - 1; step++) {
        int a = pick(), b = pick();
        weight[next] = weight[a] + weight[b];
        parent[a] = parent[b] = next;
        next++;
    }
    std::vector<uint32_t> depth(2 * m - 1, 0);
    for (int v = 2 * m - 3; v >= 0; v--) depth[v] = depth[parent[v]] + 1;
    for (int i = 0; i < m; i++) len[leaves[i].second] = depth[i];
}

// Enforce len <= L: clamp, then lengthen the deepest codes still shorter than
// L (the least frequent first) until the Kraft sum fits, then shorten the most
// frequent codes while the slack allows. Kraft sums in units of 2^-L.
void limit_lengths(const uint64_t counts[256], uint32_t len[256], uint32_t L) {
    uint32_t maxl = 0;
    for (int s = 0; s < 256; s++) maxl = std::max(maxl, len[s]);
    if (maxl <= L) return;
    const uint64_t target = 1ull << L;
    uint64_t K = 0;
    for (int s = 0; s < 256; s++)
        if (len[s]) {
            len[s] = std::min(len[s], L);
            K += 1ull << (L - len[s]);
        }
    while (K > target) {
        int best = -1;
        for (int s = 0; s < 256; s++)
            if (len[s] && len[s] < L &&
                (best < 0 || len[s] > len[best] || (len[s] == len[best] && counts[s] < counts[best])))
                best = s;
        K -= 1ull << (L - len[best] - 1);
        len[best]++;
    }
    for (;;) {
        int best = -1;
        for (int s = 0; s < 256; s++)
            if (len[s] > 1 && K + (1ull << (L - len[s])) <= target &&
                (best < 0 || counts[s] > counts[best]))
                best = s;
        if (best < 0) break;
        K += 1ull << (L - len[best]);
        len[best]--;
    }
}

// Canonical codewords: (length, symbol) order, consecutive values, shifted
// left whenever the length grows (the RFC 1951 section 3.2.2 rule).
void canonical(const uint32_t len[256], uint32_t code[256], std::vector<int> &order) {
    order.clear();
    for (int s = 0; s < 256; s++)
        if (len[s]) order.push_back(s);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return len[a] < len[b]; });
    uint32_t c = 0, prev = 0;
    for (size_t i = 0; i < order.size(); i++) {
        int s = order[i];
        if (i) c = (c + 1) << (len[s] - prev);
        code[s] = c;
        prev = len[s];
    }
}

// Hierarchical 256-entry tables indexed by successive 8-bit slices of a code.
bool build_tables(const uint32_t len[256], const uint32_t code[256], const std::vector<int> &order,
                  std::vector<uint16_t> &tables) {
    tables.assign(256, 0xFFFF);
    for (int s : order) {
        uint32_t l = len[s], c = code[s], t = 0, depth = 0;
        while (l > 8 * (depth + 1)) {
            uint32_t slice = (c >> (l - 8 * (depth + 1))) & 0xFF;
            uint16_t &e = tables[t * 256 + slice];
            if (e == 0xFFFF) {
                uint32_t nt = (uint32_t)(tables.size() / 256);
                if (nt >= kMaxTables) return false;
                e = (uint16_t)(0x8000 | nt);
                tables.resize(tables.size() + 256, 0xFFFF);
            }
            t = tables[t * 256 + slice] & 0x7FFF;
            depth++;
        }
        uint32_t rest = l - 8 * depth;
        uint32_t first = (c & ((1u << rest) - 1)) << (8 - rest);
        for (uint32_t f = 0; f < (1u << (8 - rest)); f++)
            tables[t * 256 + first + f] = (uint16_t)((l << 8) | (uint32_t)s);
    }
    return true;
}

lwc_status check_args(const uint16_t *src, uint64_t n, lwc_desc *desc, void **blob, uint64_t *bytes) {
    if (!desc || !blob || !bytes) return fail(LWC_ERR_INVALID_ARG, "NULL output pointer");
    if (n && !src) return fail(LWC_ERR_INVALID_ARG, "NULL source with n > 0");
    if (n > (1ull << 40)) return fail(LWC_ERR_INVALID_ARG, "n too large");
    return LWC_OK;
}

}  // namespace

// ------------------------------------------------------------ blob plans

lwc_status check_df11_params(uint32_t C, uint32_t T, uint32_t L) {
    if (C % 4 || C < 8 || C > 1024 || T % 32 || T < 32 || T > 1024 || L < 9 || L > kFormatMaxLen)
        return fail(LWC_ERR_INVALID_ARG, "bad DFloat11 parameters (chunk %u, block %u, max_len %u)", C, T, L);
    return LWC_OK;
}

uint64_t lo_section_bytes(uint32_t elem, uint64_t n) {
    if (elem == LWC_ELEM_FP32) return round_up(2 * n, 16);
    if (elem == LWC_ELEM_FP16) return round_up((3 * n + 7) / 8 + 16, 16);
    return 0;
}

lwc_status plan_dfloat11(const uint64_t counts[256], uint64_t n, uint32_t C, uint32_t T, uint32_t L,
                         bool chunk_counts, Df11Plan &p, uint64_t lo_bytes) {
    if (lwc_status st = check_df11_params(C, T, L)) return st;
    int present = 0, only = 0;
    for (int s = 0; s < 256; s++)
        if (counts[s]) present++, only = s;
    lwc_desc &d = p.d;
    std::memset(&d, 0, sizeof d);
    d.magic = kMagic;
    d.version = kVersion;
    d.codec = LWC_CODEC_DFLOAT11;
    d.n = n;
    d.chunk_bytes = C;
    d.threads_per_block = T;
    std::memset(p.len, 0, sizeof p.len);
    std::memset(p.code, 0, sizeof p.code);
    p.tables.clear();
    p.single = present < 2;
    if (!p.single) {
        std::vector<int> order;
        huffman_lengths(counts, p.len);
        limit_lengths(counts, p.len, L);
        canonical(p.len, p.code, order);
        if (!build_tables(p.len, p.code, order, p.tables))
            return fail(LWC_ERR_UNSUPPORTED, "code needs more than %u lookup tables", kMaxTables);
        for (int s = 0; s < 256; s++) {
            d.total_bits += counts[s] * p.len[s];
            d.max_len = std::max(d.max_len, p.len[s]);
        }
        d.n_tables = (uint32_t)(p.tables.size() / 256);
        const uint64_t cb = 8ull * C;
        d.n_chunks = (d.total_bits + cb - 1) / cb;
        d.n_blocks = (d.n_chunks + T - 1) / T;
        d.stream_bytes = round_up(4 * ((d.total_bits + 31) / 32) + 16, 16);
        // codes are at least min_len bits, so at most ceil(cb / min_len) start in a chunk
        uint32_t min_len = 32;
        for (int s = 0; s < 256; s++)
            if (p.len[s]) min_len = std::min(min_len, p.len[s]);
        if (chunk_counts && (cb + min_len - 1) / min_len <= 255) d.flags |= kFlagChunkCounts;
    } else {
        d.flags = n ? kFlagSingleExponent : 0;
        d.const_exp = (uint32_t)only;
    }
    BlobLayout lay;
    d.off_lengths = lay.place(256);
    d.off_lut = lay.place(2 * p.tables.size());
    d.off_gaps = lay.place(d.n_blocks * T);
    if (d.flags & kFlagChunkCounts) d.off_counts = lay.place(d.n_blocks * T);
    d.off_blkoff = lay.place(8 * (d.n_blocks + 1));
    d.off_stream = lay.place(d.stream_bytes);
    d.off_sm = lay.place(round_up(n, 16));
    if (lo_bytes) {
        d.off_lo = lay.place(lo_bytes);
        d.lo_bytes = lo_bytes;
    }
    d.total_bytes = lay.total();
    return LWC_OK;
}

void codebook_layout(uint32_t U, uint64_t n, lwc_desc &d) {
    std::memset(&d, 0, sizeof d);
    d.magic = kMagic;
    d.version = kVersion;
    d.codec = LWC_CODEC_CODEBOOK;
    d.n = n;
    d.U = U;
    while ((1ull << d.k) < d.U) d.k++;
    d.packed_bytes = d.k ? round_up((n * d.k + 7) / 8 + 16, 16) : 0;
    BlobLayout lay;
    d.off_table = lay.place(2ull * d.U);
    d.off_packed = lay.place(d.packed_bytes);
    d.total_bytes = lay.total();
}

void plan_codebook(const std::vector<uint8_t> &seen, uint64_t n, CbPlan &p) {
    p.table.clear();
    p.rank.assign(65536, 0);
    for (uint32_t v = 0; v < 65536; v++)
        if (seen[v]) {
            p.rank[v] = (uint16_t)p.table.size();
            p.table.push_back((uint16_t)v);
        }
    codebook_layout((uint32_t)p.table.size(), n, p.d);
}

// ------------------------------------------------------- descriptor checks

static bool inside(uint64_t off, uint64_t bytes, uint64_t total) {
    return off % 16 == 0 && off >= kHeaderBytes && off <= total && bytes <= total - off;
}

lwc_status check_df11_desc(const lwc_desc *d) {
    if (!d) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    if (d->magic != kMagic || d->version != kVersion) return fail(LWC_ERR_CORRUPT, "bad magic/version");
    if (d->codec != LWC_CODEC_DFLOAT11) return fail(LWC_ERR_INVALID_ARG, "descriptor is not DFloat11");
    const uint64_t T = d->threads_per_block, C = d->chunk_bytes, tot = d->total_bytes;
    if (C % 4 || C < 8 || C > 1024 || T % 32 || T < 32 || T > 1024)
        return fail(LWC_ERR_CORRUPT, "bad chunk_bytes/threads_per_block (%llu, %llu)",
                    (unsigned long long)C, (unsigned long long)T);
    if (!inside(d->off_sm, round_up(d->n, 16), tot) || !inside(d->off_lengths, 256, tot))
        return fail(LWC_ERR_CORRUPT, "sign/mantissa or lengths section outside the blob");
    if (d->elem > LWC_ELEM_FP16) return fail(LWC_ERR_CORRUPT, "unknown element type %u", d->elem);
    if (d->elem != LWC_ELEM_BF16 && d->n) {
        const uint64_t need = d->elem == LWC_ELEM_FP32 ? 2 * d->n : (3 * d->n + 7) / 8 + 8;
        if (d->lo_bytes < need || !inside(d->off_lo, d->lo_bytes, tot))
            return fail(LWC_ERR_CORRUPT, "low-mantissa section too short or outside the blob");
    }
    if (d->n == 0 || (d->flags & kFlagSingleExponent)) {
        if (d->const_exp > 255) return fail(LWC_ERR_CORRUPT, "bad const_exp");
        return LWC_OK;
    }
    if (d->max_len < 1 || d->max_len > kFormatMaxLen) return fail(LWC_ERR_CORRUPT, "bad max_len");
    if (d->n_tables < 1 || d->n_tables > kMaxTables) return fail(LWC_ERR_CORRUPT, "bad n_tables");
    const uint64_t cb = 8 * C;
    if (d->total_bits == 0 || d->n_chunks != (d->total_bits + cb - 1) / cb ||
        d->n_blocks != (d->n_chunks + T - 1) / T)
        return fail(LWC_ERR_CORRUPT, "chunk/block counts inconsistent with total_bits");
    if (d->total_bits > 32ull * d->n || d->total_bits < d->n)
        return fail(LWC_ERR_CORRUPT, "total_bits outside [n, 32 n]");
    if (d->stream_bytes % 16 || d->stream_bytes < 4 * ((d->total_bits + 31) / 32) + 16)
        return fail(LWC_ERR_CORRUPT, "stream section too short");
    if (d->max_block_count == 0 || d->max_block_count > T * cb || d->max_block_count > d->n)
        return fail(LWC_ERR_CORRUPT, "bad max_block_count");
    if ((d->flags & kFlagChunkCounts) && !inside(d->off_counts, d->n_blocks * T, tot))
        return fail(LWC_ERR_CORRUPT, "chunk-count section outside the blob");
    if (!inside(d->off_lut, 512ull * d->n_tables, tot) || !inside(d->off_gaps, d->n_blocks * T, tot) ||
        !inside(d->off_blkoff, 8 * (d->n_blocks + 1), tot) || !inside(d->off_stream, d->stream_bytes, tot))
        return fail(LWC_ERR_CORRUPT, "section outside the blob");
    if (d->n_blocks > 0xFFFFFFFFull) return fail(LWC_ERR_UNSUPPORTED, "too many blocks");
    return LWC_OK;
}

lwc_status check_codebook_desc(const lwc_desc *d) {
    if (!d) return fail(LWC_ERR_INVALID_ARG, "NULL descriptor");
    if (d->magic != kMagic || d->version != kVersion) return fail(LWC_ERR_CORRUPT, "bad magic/version");
    if (d->codec != LWC_CODEC_CODEBOOK) return fail(LWC_ERR_INVALID_ARG, "descriptor is not codebook");
    if (d->n == 0) return LWC_OK;
    if (d->U < 1 || d->U > 65536 || d->k > 16 || (1ull << d->k) < d->U || (d->k && (1ull << (d->k - 1)) >= d->U))
        return fail(LWC_ERR_CORRUPT, "bad U/k (%u, %u)", d->U, d->k);
    if (!inside(d->off_table, 2ull * d->U, d->total_bytes)) return fail(LWC_ERR_CORRUPT, "table outside the blob");
    if (d->k) {
        if (d->packed_bytes % 16 || d->packed_bytes < (d->n * d->k + 7) / 8 + 16)
            return fail(LWC_ERR_CORRUPT, "packed section too short");
        if (!inside(d->off_packed, d->packed_bytes, d->total_bytes))
            return fail(LWC_ERR_CORRUPT, "packed section outside the blob");
    }
    return LWC_OK;
}

// The DFloat11 encoder proper, on BF16-shaped 16-bit patterns; for FP32 and
// FP16 elements `lo` holds the raw low-mantissa section (lo_len bytes) and
// `elem` is recorded in the header.
lwc_status encode_df11(const uint16_t *src, uint64_t n, const lwc_df11_params *params, uint32_t elem,
                       const uint8_t *lo, uint64_t lo_len, lwc_desc *desc_out, void **blob_out, uint64_t *bytes_out) {
    lwc_status st;
    const uint32_t C = params ? params->chunk_bytes : kDefaultChunkBytes;
    const uint32_t T = params ? params->threads_per_block : kDefaultThreadsPerBlock;
    const uint32_t L = params ? params->max_len : kDefaultMaxLen;
    const bool with_counts = params ? params->chunk_counts != 0 : kDefaultChunkCounts != 0;

    // exponent histogram, then the code and the section layout
    uint64_t counts[256] = {0};
    for (uint64_t i = 0; i < n; i++) counts[(src[i] >> 7) & 0xFF]++;
    Df11Plan plan;
    st = plan_dfloat11(counts, n, C, T, L, with_counts, plan, lo_section_bytes(elem, n));
    if (st) return st;
    plan.d.elem = elem;
    lwc_desc &d = plan.d;
    const bool present2 = !plan.single;
    const uint32_t *len = plan.len, *code = plan.code;
    const std::vector<uint16_t> &tables = plan.tables;

    uint8_t *blob = (uint8_t *)std::calloc(1, d.total_bytes);
    if (!blob) return fail(LWC_ERR_NOMEM, "cannot allocate %llu bytes", (unsigned long long)d.total_bytes);

    for (int s = 0; s < 256; s++) blob[d.off_lengths + s] = (uint8_t)len[s];
    if (!tables.empty()) std::memcpy(blob + d.off_lut, tables.data(), 2 * tables.size());

    // sign|mantissa bytes
    uint8_t *sm = blob + d.off_sm;
    for (uint64_t i = 0; i < n; i++) sm[i] = (uint8_t)(((src[i] >> 8) & 0x80) | (src[i] & 0x7F));

    if (present2) {
        // codes, MSB first in u32 words, with chunk gaps, block offsets and
        // (when planned) per-chunk code counts
        uint32_t *words = reinterpret_cast<uint32_t *>(blob + d.off_stream);
        uint8_t *gaps = blob + d.off_gaps;
        uint8_t *ccount = (d.flags & kFlagChunkCounts) ? blob + d.off_counts : nullptr;
        uint64_t *blkoff = reinterpret_cast<uint64_t *>(blob + d.off_blkoff);
        uint64_t lut32[256];  // (len << 32) | code
        for (int s = 0; s < 256; s++) lut32[s] = ((uint64_t)len[s] << 32) | code[s];
        const uint64_t cb = 8ull * C, bb = cb * T;
        uint64_t pos = 0, acc = 0, next_chunk_bit = 0, next_block_bit = 0, chunk = 0, block = 0;
        uint32_t nacc = 0;
        uint64_t wi = 0;
        for (uint64_t i = 0; i < n; i++) {
            if (pos >= next_chunk_bit) {
                while (chunk < d.n_chunks && chunk * cb <= pos) {
                    gaps[chunk] = (uint8_t)(pos - chunk * cb);
                    chunk++;
                }
                next_chunk_bit = chunk * cb;
                if (pos >= next_block_bit) {
                    while (block < d.n_blocks && block * bb <= pos) blkoff[block++] = i;
                    next_block_bit = block < d.n_blocks ? block * bb : ~0ull;
                }
                if (chunk >= d.n_chunks) next_chunk_bit = ~0ull;
            }
            if (ccount) ccount[chunk - 1]++;   // this code starts in chunk `chunk - 1`
            const uint64_t lc = lut32[(src[i] >> 7) & 0xFF];
            const uint32_t l = (uint32_t)(lc >> 32);
            acc = (acc << l) | (uint32_t)lc;
            nacc += l;
            pos += l;
            if (nacc >= 32) {
                nacc -= 32;
                words[wi++] = (uint32_t)(acc >> nacc);
            }
        }
        if (nacc) words[wi++] = (uint32_t)(acc << (32 - nacc));
        for (; chunk < d.n_chunks; chunk++) gaps[chunk] = (uint8_t)(d.total_bits - chunk * cb);
        for (; block < d.n_blocks; block++) blkoff[block] = n;
        blkoff[d.n_blocks] = n;
        uint64_t mx = 0;
        for (uint64_t b = 0; b < d.n_blocks; b++) mx = std::max(mx, blkoff[b + 1] - blkoff[b]);
        d.max_block_count = (uint32_t)mx;
        if (pos != d.total_bits) {
            std::free(blob);
            return fail(LWC_ERR_CORRUPT, "internal: bit count mismatch");
        }
    }
    if (lo_len) std::memcpy(blob + d.off_lo, lo, lo_len);
    write_header(blob, d);
    *desc_out = d;
    *blob_out = blob;
    *bytes_out = d.total_bytes;
    clear_error();
    return LWC_OK;
}

}  // namespace lwc

using namespace lwc;

extern "C" {

lwc_status lwc_encode_dfloat11(const uint16_t *src, uint64_t n, const lwc_df11_params *params,
                               lwc_desc *desc_out, void **blob_out, uint64_t *bytes_out) {
    lwc_status st = check_args(src, n, desc_out, blob_out, bytes_out);
    if (st) return st;
    return encode_df11(src, n, params, LWC_ELEM_BF16, nullptr, 0, desc_out, blob_out, bytes_out);
}

lwc_status lwc_encode_dfloat11_elements(const void *src, uint64_t n, uint32_t elem, const lwc_df11_params *params,
                                        lwc_desc *desc_out, void **blob_out, uint64_t *bytes_out) {
    lwc_status st = check_args(static_cast<const uint16_t *>(src), n, desc_out, blob_out, bytes_out);
    if (st) return st;
    if (elem == LWC_ELEM_BF16)
        return encode_df11(static_cast<const uint16_t *>(src), n, params, elem, nullptr, 0, desc_out, blob_out,
                           bytes_out);
    if (elem != LWC_ELEM_FP32 && elem != LWC_ELEM_FP16) return fail(LWC_ERR_INVALID_ARG, "unknown element type %u", elem);
    // BF16-shaped patterns + raw low mantissa bits
    std::vector<uint16_t> v(n);
    std::vector<uint8_t> lo;
    if (elem == LWC_ELEM_FP32) {
        const uint32_t *x = static_cast<const uint32_t *>(src);
        lo.resize(2 * n);
        for (uint64_t i = 0; i < n; i++) {
            v[i] = (uint16_t)(x[i] >> 16);
            const uint16_t l = (uint16_t)x[i];
            std::memcpy(&lo[2 * i], &l, 2);
        }
    } else {
        const uint16_t *x = static_cast<const uint16_t *>(src);
        lo.assign((3 * n + 7) / 8, 0);
        for (uint64_t i = 0; i < n; i++) {
            const uint32_t w = x[i], mant = w & 0x3FF;
            v[i] = (uint16_t)((w & 0x8000) | (((w >> 10) & 0x1F) << 7) | (mant >> 3));
            const uint64_t b = 3 * i;   // 3 bits at stream bit b, least significant first
            const uint32_t l = mant & 7;
            lo[b >> 3] |= (uint8_t)(l << (b & 7));
            if ((b & 7) > 5) lo[(b >> 3) + 1] |= (uint8_t)(l >> (8 - (b & 7)));
        }
    }
    return encode_df11(v.data(), n, params, elem, lo.data(), lo.size(), desc_out, blob_out, bytes_out);
}

lwc_status lwc_encode_codebook(const uint16_t *src, uint64_t n, lwc_desc *desc_out, void **blob_out,
                               uint64_t *bytes_out) {
    lwc_status st = check_args(src, n, desc_out, blob_out, bytes_out);
    if (st) return st;
    std::vector<uint8_t> seen(65536, 0);
    for (uint64_t i = 0; i < n; i++) seen[src[i]] = 1;
    CbPlan plan;
    plan_codebook(seen, n, plan);
    lwc_desc &d = plan.d;
    const std::vector<uint16_t> &table = plan.table, &rank = plan.rank;
    uint8_t *blob = (uint8_t *)std::calloc(1, d.total_bytes);
    if (!blob) return fail(LWC_ERR_NOMEM, "cannot allocate %llu bytes", (unsigned long long)d.total_bytes);
    if (d.U) std::memcpy(blob + d.off_table, table.data(), 2ull * d.U);
    if (d.k) {
        uint32_t *words = reinterpret_cast<uint32_t *>(blob + d.off_packed);
        uint64_t acc = 0, wi = 0;
        uint32_t nacc = 0;
        for (uint64_t i = 0; i < n; i++) {
            acc |= (uint64_t)rank[src[i]] << nacc;
            nacc += d.k;
            if (nacc >= 32) {
                words[wi++] = (uint32_t)acc;
                acc >>= 32;
                nacc -= 32;
            }
        }
        if (nacc) words[wi++] = (uint32_t)acc;
    }
    write_header(blob, d);
    *desc_out = d;
    *blob_out = blob;
    *bytes_out = d.total_bytes;
    clear_error();
    return LWC_OK;
}

void lwc_free(void *blob) { std::free(blob); }

lwc_status lwc_desc_from_blob(const void *blob, uint64_t bytes, lwc_desc *out) {
    if (!blob || !out) return fail(LWC_ERR_INVALID_ARG, "NULL argument");
    if (bytes < kHeaderBytes) return fail(LWC_ERR_CORRUPT, "blob shorter than its header");
    const uint8_t *h = static_cast<const uint8_t *>(blob);
    if (get<uint32_t>(h, 24) != kHeaderBytes) return fail(LWC_ERR_CORRUPT, "bad header size");
    lwc_desc d;
    read_header(h, d);
    if (d.total_bytes != bytes) return fail(LWC_ERR_CORRUPT, "total_bytes %llu != blob size %llu",
                                            (unsigned long long)d.total_bytes, (unsigned long long)bytes);
    lwc_status st;
    if (d.codec == LWC_CODEC_DFLOAT11) st = check_df11_desc(&d);
    else if (d.codec == LWC_CODEC_CODEBOOK) st = check_codebook_desc(&d);
    else st = fail(LWC_ERR_CORRUPT, "unknown codec %u", d.codec);
    if (st) return st;
    *out = d;
    clear_error();
    return LWC_OK;
}

const char *lwc_status_string(lwc_status s) {
    switch (s) {
    case LWC_OK: return "ok";
    case LWC_ERR_INVALID_ARG: return "invalid argument";
    case LWC_ERR_MISALIGNED: return "misaligned device pointer";
    case LWC_ERR_CORRUPT: return "corrupt blob or descriptor";
    case LWC_ERR_UNSUPPORTED: return "unsupported";
    case LWC_ERR_NOMEM: return "out of host memory";
    case LWC_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char *lwc_last_error(void) { return g_last_error.c_str(); }

int lwc_version(void) { return 10000; }

}  // extern "C"
