// pp_build.cuh - pp_build_meta's kernels: descriptors + segment boundaries -> position ids and the tile schedule.
//
// Position ids follow "prefix_grouper_utils.py" section 1 (prefix 0..P-1; every response restarts at P). The tile
// schedule follows the "PackInfer" abstract: attention work is built directly over the packed query-key regions
// (fully masked sibling tiles are never listed) and ordered so the persistent kernels stay balanced (longest
// first).
#pragma once
#include "../../include/pp.h"
#include "pp_meta.cuh"

namespace pp {

enum DevErr : int32_t {
    DEVERR_TIMEOUT = 1,
    DEVERR_BAD_SEGMENTS = 2,   // cu_seqlens not monotone / not from 0 to T
    DEVERR_BAD_GROUPS = 4,     // descriptors disagree with the segments
    DEVERR_BAD_TOKEN = 8,      // a token id outside [0, V) given to pp_response_logprobs
};

__device__ int32_t g_dev_err;  // this device's error word, read and cleared by pp_get_status

__device__ __forceinline__ void set_dev_err(int32_t bits) { atomicOr(&g_dev_err, bits); }

// Block-wide exclusive scans of K int32 arrays of length n, in place (one block of NT threads, NT a multiple of 32
// and at most 1024, any n): warp-shuffle scans, then one scan of the warp totals, two block barriers per NT
// elements. tot[k] receives array k's total. s_tmp holds at least 32 * K ints; every thread of the block calls it.
template <int NT, int K>
__device__ void block_exclusive_scan_multi(int32_t *const (&a)[K], int n, int32_t *s_tmp, int32_t (&tot)[K]) {
    static_assert(NT % 32 == 0 && NT <= 1024, "block size");
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int32_t carry[K];
#pragma unroll
    for (int k = 0; k < K; ++k) carry[k] = 0;
    for (int base = 0; base < n; base += NT) {
        const int i = base + threadIdx.x;
        int32_t v[K], x[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            v[k] = i < n ? a[k][i] : 0;
            x[k] = v[k];
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1)
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const int32_t t = __shfl_up_sync(0xffffffffu, x[k], off);
                if (lane >= off) x[k] += t;
            }
        if (lane == 31)
#pragma unroll
            for (int k = 0; k < K; ++k) s_tmp[k * 32 + wid] = x[k];
        __syncthreads();
        if (wid == 0) {
#pragma unroll
            for (int k = 0; k < K; ++k) {
                int32_t y = lane < NW ? s_tmp[k * 32 + lane] : 0;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int32_t t = __shfl_up_sync(0xffffffffu, y, off);
                    if (lane >= off) y += t;
                }
                if (lane < NW) s_tmp[k * 32 + lane] = y;           // inclusive scan of the warp totals
            }
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int32_t before = wid > 0 ? s_tmp[k * 32 + wid - 1] : 0;
            if (i < n) a[k][i] = carry[k] + before + x[k] - v[k];
            carry[k] += s_tmp[k * 32 + NW - 1];
        }
        __syncthreads();                                           // s_tmp is rewritten by the next round
    }
#pragma unroll
    for (int k = 0; k < K; ++k) tot[k] = carry[k];
}

// One array: block_exclusive_scan_multi with K = 1; returns the total.
template <int NT>
__device__ int32_t block_exclusive_scan(int32_t *a, int n, int32_t *s_tmp) {
    int32_t *const arr[1] = {a};
    int32_t tot[1];
    block_exclusive_scan_multi<NT, 1>(arr, n, s_tmp, tot);
    return tot[0];
}

__device__ __forceinline__ int upper_bound_i32(const int32_t *a, int n, int32_t key) {
    int lo = 0, hi = n;   // first index with a[idx] > key
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] <= key) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// Stage 0: write the header (sizes and section offsets computed on the host) into the metadata buffer.
__global__ void k_meta_header(void *meta, MetaHeader h) { *meta_ptr<MetaHeader>(meta, 0) = h; }

// Stage 1 (one block): validate segments, group offsets, per-group tile counts and their prefix sums.
// scratch layout: [0, G+1) qtile offsets, [G+1, 2G+2) ktile offsets (reused in stage 3).
template <int NT>
__global__ void __launch_bounds__(NT) k_meta_groups(const pp_group_desc *__restrict__ groups,
                                                    const int32_t *__restrict__ cu, void *meta, int32_t *qoff,
                                                    int32_t *koff) {
    __shared__ int32_t s_tmp[NT];
    __shared__ int32_t s_bad;
    MetaHeader *h = meta_ptr<MetaHeader>(meta, 0);
    const int G = h->G, nseg = h->nseg, T = h->T;
    GroupInfo *gi = meta_ptr<GroupInfo>(meta, h->off_groups);
    int32_t *gseg = meta_ptr<int32_t>(meta, h->off_gseg);
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < nseg; i += NT)
        if (cu[i] > cu[i + 1]) atomicOr(&s_bad, DEVERR_BAD_SEGMENTS);
    if (threadIdx.x == 0 && (cu[0] != 0 || cu[nseg] != T)) atomicOr(&s_bad, DEVERR_BAD_SEGMENTS);
    for (int g = threadIdx.x; g < G; g += NT) {
        const pp_group_desc d = groups[g];
        if (d.prefix_len < 0 || d.num_suffixes < 0) atomicOr(&s_bad, DEVERR_BAD_GROUPS);
        gseg[g] = 1 + (d.num_suffixes > 0 ? d.num_suffixes : 0);
    }
    __syncthreads();
    const int32_t tot = block_exclusive_scan<NT>(gseg, G, s_tmp);
    if (threadIdx.x == 0) {
        gseg[G] = tot;
        if (tot != nseg) atomicOr(&s_bad, DEVERR_BAD_GROUPS);
    }
    __syncthreads();
    if (s_bad == 0) {
        for (int g = threadIdx.x; g < G; g += NT) {
            const int s0 = gseg[g], s1 = gseg[g + 1];
            GroupInfo x;
            x.start = cu[s0];
            x.len = cu[s1] - cu[s0];
            x.plen = cu[s0 + 1] - cu[s0];
            x.nsuf = s1 - s0 - 1;
            if (x.plen != groups[g].prefix_len) atomicOr(&s_bad, DEVERR_BAD_GROUPS);
            gi[g] = x;
            qoff[g] = (x.len + FWD_BM - 1) / FWD_BM;
            koff[g] = (x.len + BWD_BN - 1) / BWD_BN;
        }
    }
    __syncthreads();
    int32_t nq = 0, nk = 0;
    if (s_bad == 0) {
        nq = block_exclusive_scan<NT>(qoff, G, s_tmp);
        nk = block_exclusive_scan<NT>(koff, G, s_tmp);
    }
    if (threadIdx.x == 0) {
        qoff[G] = nq;
        koff[G] = nk;
        h->n_qt = nq;
        h->n_kt = nk;
        h->n_bw = 0;
        h->n_split = 0;
        h->dev_err = s_bad;
        if (s_bad) set_dev_err(s_bad);
    }
}

// Stage 2 (grid over tokens): position ids and the per-token segment table.
__global__ void k_meta_tokens(const int32_t *__restrict__ cu, void *meta, int32_t *__restrict__ pos) {
    const MetaHeader *h = meta_ptr<MetaHeader>(meta, 0);
    if (h->dev_err) return;
    const int T = h->T, nseg = h->nseg, G = h->G;
    const GroupInfo *gi = meta_ptr<GroupInfo>(meta, h->off_groups);
    const int32_t *gseg = meta_ptr<int32_t>(meta, h->off_gseg);
    int32_t *seg_start = meta_ptr<int32_t>(meta, h->off_seg_start);
    int32_t *key_end = meta_ptr<int32_t>(meta, h->off_key_end);
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
        const int s = upper_bound_i32(cu, nseg + 1, t) - 1;      // cu[s] <= t < cu[s+1]
        const int g = upper_bound_i32(gseg, G + 1, s) - 1;       // gseg[g] <= s < gseg[g+1]
        const GroupInfo x = gi[g];
        const bool prefix = (s == gseg[g]);
        pos[t] = prefix ? (t - x.start) : (x.plen + (t - cu[s]));
        seg_start[t] = cu[s];
        key_end[t] = prefix ? (x.start + x.len) : cu[s + 1];
    }
}

// Stage 3 (grid over tiles): forward query tiles and backward key tiles.
__global__ void k_meta_tiles(void *meta, const int32_t *__restrict__ qoff, const int32_t *__restrict__ koff) {
    const MetaHeader *h = meta_ptr<MetaHeader>(meta, 0);
    if (h->dev_err) return;
    const int G = h->G, nq = h->n_qt, nk = h->n_kt;
    const GroupInfo *gi = meta_ptr<GroupInfo>(meta, h->off_groups);
    const int32_t *seg_start = meta_ptr<int32_t>(meta, h->off_seg_start);
    const int32_t *key_end = meta_ptr<int32_t>(meta, h->off_key_end);
    QTile *qt = meta_ptr<QTile>(meta, h->off_qt);
    KTile *kt = meta_ptr<KTile>(meta, h->off_kt);
    const int n = nq > nk ? nq : nk;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        if (i < nq) {
            const int g = upper_bound_i32(qoff, G + 1, i) - 1;
            const GroupInfo x = gi[g];
            const int a = i - qoff[g];
            QTile t;
            t.row0 = x.start + a * FWD_BM;
            t.gstart = x.start;
            t.glen = x.len;
            t.plen = x.plen;
            t.group = g;
            t.pad0 = t.pad1 = 0;
            const int x0 = a * FWD_BM;
            const int xm = min(x0 + FWD_BM, x.len) - 1;
            t.s0first = x0 >= x.plen ? seg_start[x.start + x0] - x.start : x.plen;
            t.s0last = xm >= x.plen ? seg_start[x.start + xm] - x.start : 0;
            const bool any_resp = xm >= x.plen;
            const int a_end = any_resp ? x.plen : xm + 1;
            t.nA = (a_end + FWD_BN - 1) / FWD_BN;
            t.bB = 0;
            t.eB = 0;
            if (any_resp) {
                const int b_start = x0 >= x.plen ? t.s0first : x.plen;
                int bB = b_start / FWD_BN, eB = xm / FWD_BN + 1;
                if (bB <= t.nA) {            // the two runs touch: merge into one
                    t.nA = max(t.nA, eB);
                } else {
                    t.bB = bB;
                    t.eB = eB;
                }
            }
            qt[i] = t;
        }
        if (i < nk) {
            const int g = upper_bound_i32(koff, G + 1, i) - 1;
            const GroupInfo x = gi[g];
            const int b = i - koff[g];
            KTile t;
            t.row0 = x.start + b * BWD_BN;
            t.gstart = x.start;
            t.glen = x.len;
            t.plen = x.plen;
            t.group = g;
            const int y0 = b * BWD_BN;
            const int ylast = min(y0 + BWD_BN, x.len) - 1;
            const int e = y0 < x.plen ? x.len : key_end[x.start + ylast] - x.start;
            t.qa = y0 / BWD_BM;
            t.qb = (e + BWD_BM - 1) / BWD_BM;
            const int nqt = t.qb - t.qa;
            int c = (nqt + BWD_CHUNK_QTILES - 1) / BWD_CHUNK_QTILES;
            t.nch = c < 1 ? 1 : (c > BWD_MAX_CHUNKS ? BWD_MAX_CHUNKS : c);
            kt[i] = t;
        }
    }
}

// Stage 4 (one block): cost-ordered forward tiles and backward work chunks (counting sort, longest first).
template <int NT>
__global__ void __launch_bounds__(NT) k_meta_sort(void *meta, int32_t *chunk_off, BWork *bw_tmp) {
    __shared__ int32_t s_tmp[32];
    __shared__ int32_t s_hist[SORT_BINS];
    __shared__ int32_t s_nsplit;
    MetaHeader *h = meta_ptr<MetaHeader>(meta, 0);
    if (h->dev_err) return;
    if (threadIdx.x == 0) s_nsplit = 0;
    const int nq = h->n_qt, nk = h->n_kt;
    const QTile *qt = meta_ptr<QTile>(meta, h->off_qt);
    const KTile *kt = meta_ptr<KTile>(meta, h->off_kt);
    int32_t *qorder = meta_ptr<int32_t>(meta, h->off_qorder);
    QTile *qts = meta_ptr<QTile>(meta, h->off_qts);
    BWork *bw = meta_ptr<BWork>(meta, h->off_bw);

    // ---- forward query tiles by decreasing key-tile count
    for (int b = threadIdx.x; b < SORT_BINS; b += NT) s_hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < nq; i += NT) atomicAdd(&s_hist[min(qtile_nkv(qt[i]), SORT_BINS - 1)], 1);
    __syncthreads();
    // descending order: bin b starts after all bins > b
    for (int b = threadIdx.x; b < SORT_BINS; b += NT) chunk_off[SORT_BINS - 1 - b] = s_hist[b];
    __syncthreads();
    block_exclusive_scan<NT>(chunk_off, SORT_BINS, s_tmp);
    for (int b = threadIdx.x; b < SORT_BINS; b += NT) s_hist[b] = chunk_off[SORT_BINS - 1 - b];
    __syncthreads();
    for (int i = threadIdx.x; i < nq; i += NT) {
        const int p = atomicAdd(&s_hist[min(qtile_nkv(qt[i]), SORT_BINS - 1)], 1);
        qorder[p] = i;
        qts[p] = qt[i];
    }
    __syncthreads();

    // ---- dS slots: one per backward step (key tile, query tile, q head of the kv head), key tiles in order
    int32_t *kslot = meta_ptr<int32_t>(meta, h->off_kslot);
    const int r = h->hq / h->hkv;
    for (int i = threadIdx.x; i <= nk; i += NT) kslot[i] = i < nk ? (kt[i].qb - kt[i].qa) * r : 0;
    __syncthreads();
    const int32_t n_slots = block_exclusive_scan<NT>(kslot, nk + 1, s_tmp);
    if (threadIdx.x == 0) h->n_slots = n_slots;

    // ---- backward chunks: split each key tile's query range [qa, qb) into nch near-equal chunks
    for (int i = threadIdx.x; i < nk; i += NT) chunk_off[i] = kt[i].nch;
    __syncthreads();
    const int32_t nbw = block_exclusive_scan<NT>(chunk_off, nk, s_tmp);
    int nsplit_local = 0;
    for (int i = threadIdx.x; i < nk; i += NT) {
        const KTile t = kt[i];
        const int nqt = t.qb - t.qa;
        if (t.nch > 1) ++nsplit_local;
        for (int c = 0; c < t.nch; ++c) {
            BWork w;
            w.kt = i;
            w.qa = t.qa + (nqt * c) / t.nch;
            w.qb = t.qa + (nqt * (c + 1)) / t.nch;
            w.split = t.nch > 1 ? 1 : 0;
            w.row0 = t.row0;
            w.gstart = t.gstart;
            w.glen = t.glen;
            w.slot0 = kslot[i] + (w.qa - t.qa) * r;
            bw_tmp[chunk_off[i] + c] = w;
        }
    }
    if (nsplit_local) atomicAdd(&s_nsplit, nsplit_local);
    for (int b = threadIdx.x; b < SORT_BINS; b += NT) s_hist[b] = 0;
    __syncthreads();
    if (threadIdx.x == 0) {
        h->n_split = s_nsplit;
        h->n_bw = nbw;
    }
    for (int i = threadIdx.x; i < nbw; i += NT) atomicAdd(&s_hist[min(bw_tmp[i].qb - bw_tmp[i].qa, SORT_BINS - 1)], 1);
    __syncthreads();
    for (int b = threadIdx.x; b < SORT_BINS; b += NT) chunk_off[SORT_BINS - 1 - b] = s_hist[b];
    __syncthreads();
    block_exclusive_scan<NT>(chunk_off, SORT_BINS, s_tmp);
    for (int b = threadIdx.x; b < SORT_BINS; b += NT) s_hist[b] = chunk_off[SORT_BINS - 1 - b];
    __syncthreads();
    for (int i = threadIdx.x; i < nbw; i += NT) {
        const BWork w = bw_tmp[i];
        const int p = atomicAdd(&s_hist[min(w.qb - w.qa, SORT_BINS - 1)], 1);
        bw[p] = w;
    }
}

// pp_meta_tiles: expand the schedule into (q_row0, kv_row0, class) triples with the kernels' own class rule.
__global__ void k_meta_expand(const void *meta, int which, int32_t *__restrict__ out, int64_t cap,
                              int32_t *__restrict__ count) {
    const MetaHeader *h = meta_ptr<MetaHeader>(meta, 0);
    if (h->dev_err) return;
    const int32_t *seg_start = meta_ptr<int32_t>(meta, h->off_seg_start);
    if (which == 0) {
        const QTile *qt = meta_ptr<QTile>(meta, h->off_qt);
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < h->n_qt; i += gridDim.x * blockDim.x) {
            const QTile t = qt[i];
            const int n = qtile_nkv(t);
            const int x0 = t.row0 - t.gstart;
            for (int j = 0; j < n; ++j) {
                const int y0 = qtile_kv(t, j) * FWD_BN;
                const int c = tile_class(x0, FWD_BM, y0, FWD_BN, t.glen, t.plen, t.s0first, t.s0last);
                const int p = atomicAdd(count, 1);
                if (p < cap) {
                    out[3 * int64_t(p)] = t.row0;
                    out[3 * int64_t(p) + 1] = t.gstart + y0;
                    out[3 * int64_t(p) + 2] = c;
                }
            }
        }
    } else {
        const KTile *kt = meta_ptr<KTile>(meta, h->off_kt);
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < h->n_kt; i += gridDim.x * blockDim.x) {
            const KTile t = kt[i];
            const int y0 = t.row0 - t.gstart;
            for (int a = t.qa; a < t.qb; ++a) {
                const int x0 = a * BWD_BM;
                const int xm = min(x0 + BWD_BM, t.glen) - 1;
                const int s0f = x0 >= t.plen ? seg_start[t.gstart + x0] - t.gstart : t.plen;
                const int s0l = xm >= t.plen ? seg_start[t.gstart + xm] - t.gstart : 0;
                const int c = tile_class(x0, BWD_BM, y0, BWD_BN, t.glen, t.plen, s0f, s0l);
                const int p = atomicAdd(count, 1);
                if (p < cap) {
                    out[3 * int64_t(p)] = t.gstart + x0;
                    out[3 * int64_t(p) + 1] = t.row0;
                    out[3 * int64_t(p) + 2] = c;
                }
            }
        }
    }
}

// pp_meta_schedule: expand the work lists the kernels execute, in their stored order, into records
// (item, q_row0, kv_row0, class, split). Forward: item = position of the query tile in the cost order (qts), one
// record per key tile it visits, split = 0. Backward: item = index of the work chunk (BWork) in its stored order, one
// record per query tile of its range, split = the chunk's flag.
__global__ void k_meta_schedule(const void *meta, int which, int32_t *__restrict__ out, int64_t cap,
                                int32_t *__restrict__ count) {
    const MetaHeader *h = meta_ptr<MetaHeader>(meta, 0);
    if (h->dev_err) return;
    const int32_t *seg_start = meta_ptr<int32_t>(meta, h->off_seg_start);
    auto emit = [&](int item, int q0, int k0, int c, int split) {
        const int p = atomicAdd(count, 1);
        if (p < cap) {
            int32_t *o = out + 5 * int64_t(p);
            o[0] = item; o[1] = q0; o[2] = k0; o[3] = c; o[4] = split;
        }
    };
    if (which == 0) {
        const QTile *qts = meta_ptr<QTile>(meta, h->off_qts);
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < h->n_qt; i += gridDim.x * blockDim.x) {
            const QTile t = qts[i];
            const int n = qtile_nkv(t);
            const int x0 = t.row0 - t.gstart;
            for (int j = 0; j < n; ++j) {
                const int y0 = qtile_kv(t, j) * FWD_BN;
                emit(i, t.row0, t.gstart + y0,
                     tile_class(x0, FWD_BM, y0, FWD_BN, t.glen, t.plen, t.s0first, t.s0last), 0);
            }
        }
    } else {
        const BWork *bw = meta_ptr<BWork>(meta, h->off_bw);
        const KTile *kt = meta_ptr<KTile>(meta, h->off_kt);
        for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < h->n_bw; i += gridDim.x * blockDim.x) {
            const BWork w = bw[i];
            const KTile t = kt[w.kt];
            const int y0 = w.row0 - w.gstart;
            for (int a = w.qa; a < w.qb; ++a) {
                const int x0 = a * BWD_BM;
                const int xm = min(x0 + BWD_BM, w.glen) - 1;
                const int s0f = x0 >= t.plen ? seg_start[w.gstart + x0] - w.gstart : t.plen;
                const int s0l = xm >= t.plen ? seg_start[w.gstart + xm] - w.gstart : 0;
                emit(i, w.gstart + x0, w.row0, tile_class(x0, BWD_BM, y0, BWD_BN, w.glen, t.plen, s0f, s0l), w.split);
            }
        }
    }
}

}  // namespace pp
