// pp_meta.cuh - layout of the metadata buffer and the tile rules shared by every kernel.
//
// Tiles are aligned to each group's start. The forward pass walks query tiles of FWD_BM rows against key tiles of
// FWD_BN rows; the backward pass walks key tiles of BWD_BN rows against query tiles of BWD_BM rows. For a group with
// prefix length P and length L (in-group offsets x for queries, y for keys) the allowed set of query x is
//     prefix row  (x <  P): keys [0, x]
//     response row(x >= P): keys [0, P) U [s0(x), x], s0(x) = first offset of x's response
// ("Preference Packing" method digest: the prompt's attention is computed once and reused by every response;
// "prefix_grouper_utils.py" diagram: every response continues the prefix on its own). Seen from key y, the queries
// that attend it form one interval [y, e(y)) with e(y) = L for a prefix key and the end of y's response otherwise.
#pragma once
#include <cstdint>

namespace pp {

constexpr int FWD_BM = 128;
constexpr int FWD_BN = 128;
constexpr int BWD_BN = 128;   // key rows per backward tile (the MMA M dimension)
constexpr int BWD_BM = 128;   // query rows per backward step (the MMA N dimension)
constexpr int BWD_MAX_CHUNKS = 16;
constexpr int BWD_CHUNK_QTILES = 8;    // target query tiles per backward work chunk (before the cap)
constexpr int SORT_BINS = 4096;
constexpr int32_t META_MAGIC = 0x314d5050;  // "PPM1"

enum TileClass : int32_t { TILE_EMPTY = 0, TILE_FULL = 1, TILE_PARTIAL = 2 };

struct alignas(16) GroupInfo {
    int32_t start;   // packed offset of the group
    int32_t len;     // L_g
    int32_t plen;    // P_g
    int32_t nsuf;    // k_g
};

struct alignas(16) QTile {      // forward query tile
    int32_t row0;     // packed row of the first query row
    int32_t gstart;   // packed offset of its group
    int32_t glen;     // group length
    int32_t plen;     // prefix length
    int32_t s0first;  // in-group start of the response of the first response row (P if the tile starts in the prefix)
    int32_t s0last;   // in-group start of the segment of the last in-group row (0 for a prefix row)
    int32_t nA;       // key tiles [0, nA) form the first run
    int32_t bB;       // key tiles [bB, eB) form the second run (empty when bB >= eB)
    int32_t eB;
    int32_t group;
    int32_t pad0, pad1;
};

struct alignas(16) KTile {      // backward key tile
    int32_t row0;
    int32_t gstart;
    int32_t glen;
    int32_t plen;
    int32_t qa, qb;   // query tiles (BWD_BM rows, in-group index) [qa, qb) attend this key tile
    int32_t nch;      // work chunks the query range is split into
    int32_t group;
};

struct alignas(16) BWork {      // backward work chunk: key tile kt, query tiles [qa, qb)
    int32_t kt;
    int32_t qa, qb;
    int32_t split;    // 1 if the key tile is split over several chunks (partials are added into fp32 scratch)
    int32_t row0, gstart, glen;   // the key tile's first row, group offset and group length (copied from kt)
    int32_t slot0;    // dS slot of the chunk's first step (query tile qa, the first q head of the kv head)
};

struct alignas(16) MetaHeader {
    int32_t magic;
    int32_t T, G, nseg, hq, hkv;
    int32_t n_qt;        // forward query tiles
    int32_t n_kt;        // backward key tiles
    int32_t n_bw;        // backward work chunks
    int32_t n_split;     // key tiles split over several chunks
    int32_t cap_qt, cap_kt, cap_bw;
    int32_t dev_err;     // non-zero if the builder found inconsistent input
    int32_t n_slots;     // backward steps (key tile, query tile, q head): one dS tile each when dS is kept
    int32_t pad;
    int64_t off_seg_start;   // int32[T]: packed start of each token's segment
    int64_t off_key_end;     // int32[T]: packed end of the query interval that attends each token as a key
    int64_t off_groups;      // GroupInfo[G]
    int64_t off_gseg;        // int32[G+1]: first segment index of each group
    int64_t off_qt;          // QTile[cap_qt], in group order
    int64_t off_qorder;      // int32[cap_qt]: query tiles sorted by decreasing cost
    int64_t off_qts;         // QTile[cap_qt]: the query tiles in that order (one load per work item)
    int64_t off_kt;          // KTile[cap_kt]
    int64_t off_bw;          // BWork[cap_bw], sorted by decreasing cost
    int64_t off_kslot;       // int32[cap_kt + 1]: first dS slot of each key tile (steps in tile order, then total)
    int64_t off_kfirst;      // int32[G + 1]: first key tile of each group (inside the builder scratch, kept)
    int64_t off_scratch;     // builder scratch: qoff int32[G+1], koff int32[G+1], tmp int32[max(cap_kt, SORT_BINS)]
    int64_t off_bw_tmp;      // builder scratch: BWork[cap_bw] before sorting
    int64_t total_bytes;
};

__host__ __device__ inline int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Section offsets: a pure function of the sizes, used by pp_meta_bounds and pp_build_meta alike.
__host__ __device__ inline MetaHeader meta_layout(int64_t T, int32_t G, int32_t nseg, int32_t hq, int32_t hkv) {
    MetaHeader h{};
    h.magic = META_MAGIC;
    h.T = static_cast<int32_t>(T);
    h.G = G;
    h.nseg = nseg;
    h.hq = hq;
    h.hkv = hkv;
    h.cap_qt = static_cast<int32_t>((T + FWD_BM - 1) / FWD_BM + G);
    h.cap_kt = static_cast<int32_t>((T + BWD_BN - 1) / BWD_BN + G);
    h.cap_bw = h.cap_kt * BWD_MAX_CHUNKS;
    int64_t o = align256(sizeof(MetaHeader));
    h.off_seg_start = o; o = align256(o + 4 * T);
    h.off_key_end = o;   o = align256(o + 4 * T);
    h.off_groups = o;    o = align256(o + int64_t(sizeof(GroupInfo)) * G);
    h.off_gseg = o;      o = align256(o + 4 * int64_t(G + 1));
    h.off_qt = o;        o = align256(o + int64_t(sizeof(QTile)) * h.cap_qt);
    h.off_qorder = o;    o = align256(o + 4 * int64_t(h.cap_qt));
    h.off_qts = o;       o = align256(o + int64_t(sizeof(QTile)) * h.cap_qt);
    h.off_kt = o;        o = align256(o + int64_t(sizeof(KTile)) * h.cap_kt);
    h.off_bw = o;        o = align256(o + int64_t(sizeof(BWork)) * h.cap_bw);
    h.off_kslot = o;     o = align256(o + 4 * int64_t(h.cap_kt + 1));
    h.off_scratch = o;
    h.off_kfirst = o + 4 * int64_t(G + 1);       // the builder's koff, written by k_meta_groups and never reused
    o = align256(o + 4 * (2 * int64_t(G + 1) + (h.cap_kt > SORT_BINS ? h.cap_kt : SORT_BINS)));
    h.off_bw_tmp = o;    o = align256(o + int64_t(sizeof(BWork)) * h.cap_bw);
    h.total_bytes = o;
    return h;
}

template <typename T>
__host__ __device__ inline T *meta_ptr(void *base, int64_t off) {
    return reinterpret_cast<T *>(reinterpret_cast<char *>(base) + off);
}
template <typename T>
__host__ __device__ inline const T *meta_ptr(const void *base, int64_t off) {
    return reinterpret_cast<const T *>(reinterpret_cast<const char *>(base) + off);
}

// Class of the tile (query rows [x0, x0+bm), key rows [y0, y0+bn)), in-group offsets, of a group of length L with
// prefix P. s0first: start of the response of the tile's first response row (P when the tile begins in the prefix);
// s0last: start of the segment of its last in-group row (0 for a prefix row). Positions past the group's end are
// not allowed, so a tile that sticks out of its group is never FULL.
__host__ __device__ inline int tile_class(int x0, int bm, int y0, int bn, int L, int P, int s0first, int s0last) {
    if (x0 >= L || y0 >= L) return TILE_EMPTY;
    const int xm = (x0 + bm < L ? x0 + bm : L) - 1;          // last in-group query row
    const int ylast = (y0 + bn < L ? y0 + bn : L) - 1;       // last in-group key row
    const bool any_resp = xm >= P;
    const int a_end = any_resp ? P : xm + 1;                 // union of allowed keys: [0, a_end) U [b_start, xm]
    const int b_start = any_resp ? (x0 >= P ? s0first : P) : 0x7fffffff;
    const bool hit = (y0 < a_end) || (ylast >= b_start && y0 <= xm);
    if (!hit) return TILE_EMPTY;
    const int y1 = y0 + bn;
    if (x0 + bm <= L && y1 <= L && y1 - 1 <= x0 && (y1 <= P || y0 >= s0last || s0last <= P)) return TILE_FULL;
    return TILE_PARTIAL;
}

// Number of key tiles a forward query tile visits (its cost).
__host__ __device__ inline int qtile_nkv(const QTile &t) {
    const int nb = t.eB > t.bB ? t.eB - t.bB : 0;
    return t.nA + nb;
}
// i-th key tile (in-group tile index) a forward query tile visits: run A, then run B.
__host__ __device__ inline int qtile_kv(const QTile &t, int i) { return i < t.nA ? i : t.bB + (i - t.nA); }

// Upper bound, from T alone, on the backward steps of one kv head (sum over key tiles of the query tiles that attend
// them, times r). A group of n key tiles has at most n (n + 1) / 2 (key tile, query tile) pairs; joining two groups
// of two or more tiles each never lowers the count, and groups of one tile add at most one pair per token, so
// T + N (N + 1) / 2 pairs with N = ceil(T / BWD_BN) bound any batch of T tokens.
__host__ __device__ inline int64_t bwd_steps_bound(int64_t T, int r) {
    const int64_t n = (T + BWD_BN - 1) / BWD_BN;
    return int64_t(r) * (T + n * (n + 1) / 2);
}

// Item that CTA b of a persistent grid of g CTAs takes in its round k, for items in decreasing cost order: each
// round deals the next g items, in alternating directions, so that the CTAs that took the costlier items of one
// round take the cheaper ones of the next (plain round-robin gives CTA 0 the costliest item of every round).
__host__ __device__ inline int alt_item(int k, int b, int g) { return k * g + ((k & 1) ? g - 1 - b : b); }

}  // namespace pp
