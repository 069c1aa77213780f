// pp_attn_bwd_dq.cuh - the dQ half of the backward, two ways, neither with atomics. k_bwd_dq_ds (at the end of this
// file) forms dQ from the dS tiles the dK/dV kernel kept in the workspace; k_bwd_dq, below, recomputes S and dP per
// tile when the workspace cannot hold those tiles.
//
// dQ_i = scale sum_j dS_ij k_j with dS_ij = p_ij (dO_i . v_j - D_i) and p_ij = exp(s_ij - lse_i), over the allowed
// keys j of query row i (pp_meta.cuh). A work item is (query tile of 128 rows, one q head); it walks the same key
// tiles as the forward pass (the two runs of the QTile) and owns its 128 dQ rows, so dQ is written once, in bf16,
// with no reduction across CTAs. Per key tile:
//   S  = Q K^T      (M = 128 queries, N = 128 keys)          TMEM S
//   dP = dO V^T                                               TMEM dP
//   gradient warps: P = exp2(S * scale log2 e - lse log2 e); dS = scale P (dP - D)  -> TMEM dP (bf16)
//   dQ += dS K      (A from TMEM, B = the K tile read N-major) TMEM dQ
// Here the thread owns a query row, so lse and D are per-thread constants: no per-column broadcast is needed.
// Recomputing S and dP costs 16 of the 24 MMAs per tile; in exchange dQ needs no fp32 accumulator and no
// reduction traffic (which measured about 6 TB/s at best on L2-resident data, below what the key-side kernel
// would otherwise need).
// Warp roles (608 threads): warps 0-15 form four gradient warpgroups, each taking 32 key columns of every tile
// (its own slice of S and dP, P kept packed in registers, its dS written into dP columns it has itself read);
// warp 16 is the TMA producer (Q and dO once per item, K through a 3-stage ring, V through a 2-stage ring); warp 17
// allocates TMEM and issues S and dP; warp 18 issues dQ.
// TMEM: S [0,128), dP/dS double-buffered [128,256) and [256,384), dQ [384,512). The second dP buffer lets dP of
// the next key tile run while dS of this one is still being formed, so the gradient warps go from P(j+1) straight
// to dS(j+1) without waiting on dQ(j).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "pp_meta.cuh"
#include "pp_ptx.cuh"
#include "pp_attn_fwd.cuh"   // bwait, FwdItem helpers

namespace pp {

constexpr int DQ_THREADS = 608;      // 16 gradient warps, producer, two MMA issuers
constexpr int DQ_KSTAGES = 3;         // K is held from S(j) (issued one tile early) to dQ(j)
constexpr int DQ_VSTAGES = 2;         // V only feeds dP(j)
constexpr int DQ_GRAD = 512;          // gradient threads (4 warpgroups x 32 key columns)
constexpr int DQ_POLY_EVERY = 4;      // one exponential pair in four on the FMA pipe (ex2_poly2), the rest on MUFU

struct DqSmem {
    static constexpr int TILE = 128 * 128 * 2;
    static constexpr int CHUNK = 128 * 64 * 2;
    alignas(1024) uint8_t q[TILE];
    alignas(1024) uint8_t dout[TILE];
    alignas(1024) uint8_t k[DQ_KSTAGES][TILE];
    alignas(1024) uint8_t v[DQ_VSTAGES][TILE];
    uint64_t q_full, q_empty, do_full, do_empty, dq_full, dq_free;
    uint64_t k_full[DQ_KSTAGES], k_empty[DQ_KSTAGES], v_full[DQ_VSTAGES], v_empty[DQ_VSTAGES];
    uint64_t s_full, s_free, dp_full[2], ds_ready[2], dq_done[2];   // ds_ready by step parity (see the gradient warps)
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(DqSmem) + 1024 <= 232448, "dQ kernel shared memory exceeds 227 KB");

struct DqItem {
    QTile t;
    int h, kh;
};

__device__ __forceinline__ DqItem dq_decode(const void *meta, const MetaHeader &hd, int item, int hq, int hkv) {
    DqItem it;
    it.t = meta_ptr<QTile>(meta, hd.off_qts)[item / hq];
    it.h = item % hq;
    it.kh = it.h / (hq / hkv);
    return it;
}

__global__ void __launch_bounds__(DQ_THREADS, 1)
k_bwd_dq(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
         const void *__restrict__ meta, const float2 *__restrict__ ldg, __nv_bfloat16 *__restrict__ dQ, int hq,
         int hkv, int64_t rows_pad, float scale, float sl2, const void *ds_buf, int64_t ds_cap) {
    extern __shared__ uint8_t smem_raw[];
    DqSmem &sm = *reinterpret_cast<DqSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
    if (ds_buf != nullptr && int64_t(hd.n_slots) * hkv <= ds_cap) return;   // dS kept: k_bwd_dq_ds computes dQ
    const int n_items = hd.n_qt * hq;
    volatile int *abort_flag = &sm.abort_flag;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, 1);
        mbar_init(&sm.do_full, 1);
        mbar_init(&sm.do_empty, 1);
        mbar_init(&sm.dq_full, 1);
        mbar_init(&sm.dq_free, DQ_GRAD);
        for (int s = 0; s < DQ_KSTAGES; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int s = 0; s < DQ_VSTAGES; ++s) {
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, DQ_GRAD);
        mbar_init(&sm.dp_full[0], 1);
        mbar_init(&sm.dp_full[1], 1);
        mbar_init(&sm.ds_ready[0], DQ_GRAD);
        mbar_init(&sm.ds_ready[1], DQ_GRAD);
        mbar_init(&sm.dq_done[0], 1);
        mbar_init(&sm.dq_done[1], 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 17) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 16 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdO);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DQ = 384;   // dP buffer b at COL_DP + 128 b

    if (hd.dev_err != 0) {
        // nothing to do: the metadata builder rejected its input
    } else if (warp == 16) {
        // ------------------------------------------------------------------ TMA producer (one thread)
        // Q and dO have their own buffers, released once the item's last S / dP is issued, so the next item's
        // tiles arrive while this one finishes; K and V come through separate rings, each freed by its last use.
        if (lane == 0) {
            uint32_t kv_it = 0, it_n = 0;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it_n) {
                const DqItem w = dq_decode(meta, hd, item, hq, hkv);
                const int n = qtile_nkv(w.t);
                if (item + int(gridDim.x) < n_items) {                 // the next item's Q and dO into L2
                    const DqItem wn = dq_decode(meta, hd, item + gridDim.x, hq, hkv);
                    for (int c = 0; c < 2; ++c) {
                        tma_prefetch_3d(&tmQ, c * 64, wn.h, wn.t.row0);
                        tma_prefetch_3d(&tmdO, c * 64, wn.h, wn.t.row0);
                    }
                }
                if (!bwait(&sm.q_empty, (it_n & 1) ^ 1, abort_flag)) goto done;
                mbar_arrive_expect_tx(&sm.q_full, DqSmem::TILE);
                for (int c = 0; c < 2; ++c)
                    tma_load_3d(sm.q + c * DqSmem::CHUNK, &tmQ, c * 64, w.h, w.t.row0, &sm.q_full);
                if (!bwait(&sm.do_empty, (it_n & 1) ^ 1, abort_flag)) goto done;
                mbar_arrive_expect_tx(&sm.do_full, DqSmem::TILE);
                for (int c = 0; c < 2; ++c)
                    tma_load_3d(sm.dout + c * DqSmem::CHUNK, &tmdO, c * 64, w.h, w.t.row0, &sm.do_full);
                for (int j = 0; j < n; ++j, ++kv_it) {
                    const int y0 = w.t.gstart + qtile_kv(w.t, j) * FWD_BN;
                    const int sk = kv_it % DQ_KSTAGES, sv = kv_it % DQ_VSTAGES;
                    if (!bwait(&sm.k_empty[sk], ((kv_it / DQ_KSTAGES) & 1) ^ 1, abort_flag)) goto done;
                    mbar_arrive_expect_tx(&sm.k_full[sk], DqSmem::TILE);
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(sm.k[sk] + c * DqSmem::CHUNK, &tmK, c * 64, w.kh, y0, &sm.k_full[sk]);
                    if (!bwait(&sm.v_empty[sv], ((kv_it / DQ_VSTAGES) & 1) ^ 1, abort_flag)) goto done;
                    mbar_arrive_expect_tx(&sm.v_full[sv], DqSmem::TILE);
                    for (int c = 0; c < 2; ++c)
                        tma_load_3d(sm.v[sv] + c * DqSmem::CHUNK, &tmV, c * 64, w.kh, y0, &sm.v_full[sv]);
                }
            }
        }
    } else if (warp == 17 || warp == 18) {
        // ------------------------------------------------------------------ MMA issuers (one thread each)
        // Issuing one MMA takes a thread about 50 cycles, close to the 64 an N = 128 MMA runs, so a single issuer
        // that also polls barriers leaves the tensor pipe idle. Warp 17 issues S and dP, warp 18 issues dQ:
        //   warp 17: S(j+1) once the gradient warps hold S(j) in registers; dP(j+1) into buffer (j+1) % 2 once dQ(j-1)
        //            has read dS(j-1) from that buffer (dq_done);
        //   warp 18: dQ(j) += dS(j) K(j) once dS(j) is in TMEM (ds_ready), then frees K(j).
        constexpr uint32_t ID_SP = idesc_bf16(128, 128, 0, 0);         // S, dP: K-major x K-major over d
        constexpr uint32_t ID_DQ = idesc_bf16(128, 128, 0, 1);         // dQ: A = dS (TMEM), B = K N-major
        constexpr uint32_t TB = DqSmem::TILE;
        const QTile *qts = meta_ptr<QTile>(meta, hd.off_qts);
        if (warp == 17 && lane == 0) {
            uint32_t kv_it = 0, it_n = 0, g = 0;                           // g: global key-tile step counter
            // descriptors built once; a stage is a constant stride away (desc_adv)
            const uint64_t q_desc = smem_desc(smem_u32(sm.q), 16, 1024);
            const uint64_t do_desc = smem_desc(smem_u32(sm.dout), 16, 1024);
            const uint64_t k_desc = smem_desc(smem_u32(sm.k[0]), 16, 1024);
            const uint64_t v_desc = smem_desc(smem_u32(sm.v[0]), 16, 1024);
            auto issue_kk = [&](uint32_t col, uint64_t a, uint64_t b) {
                const uint32_t d = tmem + col;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * DqSmem::CHUNK + (kk & 3) * 32;
                    umma_ss(d, desc_adv(a, off), desc_adv(b, off), ID_SP, kk > 0);
                }
            };
            // S of key tile `it` (ring position) into the S region; releases Q after the item's last tile
            auto issue_s = [&](uint32_t it, bool last) -> bool {
                const int sk = it % DQ_KSTAGES;
                if (!bwait(&sm.k_full[sk], (it / DQ_KSTAGES) & 1, abort_flag)) return false;
                tc_fence_after();
                issue_kk(COL_S, q_desc, k_desc + uint64_t(sk) * (TB >> 4));
                umma_commit(&sm.s_full);
                if (last) umma_commit(&sm.q_empty);
                return true;
            };
            // dP of key tile `it` into dP buffer `b`; frees its V stage, and dO after the item's last tile. Buffer b
            // last held dS(gg - 2), read by dQ(gg - 2) on the other issuer.
            auto issue_dp = [&](uint32_t it, uint32_t gg, bool last) -> bool {
                const int sv = it % DQ_VSTAGES;
                if (gg >= 2 && !bwait(&sm.dq_done[gg & 1], ((gg - 2) >> 1) & 1, abort_flag)) return false;
                if (!bwait(&sm.v_full[sv], (it / DQ_VSTAGES) & 1, abort_flag)) return false;
                tc_fence_after();
                issue_kk(COL_DP + 128 * (gg & 1), do_desc, v_desc + uint64_t(sv) * (TB >> 4));
                umma_commit(&sm.dp_full[gg & 1]);
                umma_commit(&sm.v_empty[sv]);
                if (last) umma_commit(&sm.do_empty);
                return true;
            };
            int n_next = blockIdx.x < n_items ? qtile_nkv(qts[blockIdx.x / hq]) : 0;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it_n) {
                const int n = n_next;                                  // loaded one item ahead
                if (item + int(gridDim.x) < n_items) n_next = qtile_nkv(qts[(item + gridDim.x) / hq]);
                // S and dP of the first key tile; the S region was released by s_free(g - 1)
                if (!bwait(&sm.q_full, it_n & 1, abort_flag)) goto done;
                if (g > 0 && !bwait(&sm.s_free, (g - 1) & 1, abort_flag)) goto done;
                if (!issue_s(kv_it, n == 1)) goto done;
                if (!bwait(&sm.do_full, it_n & 1, abort_flag)) goto done;
                if (!issue_dp(kv_it, g, n == 1)) goto done;
                for (int j = 0; j < n; ++j, ++kv_it, ++g) {
                    if (j + 1 < n) {
                        // the next tile's dP into the other buffer, then its S once this tile's S has been read
                        if (!issue_dp(kv_it + 1, g + 1, j + 2 == n)) goto done;
                        if (!bwait(&sm.s_free, g & 1, abort_flag)) goto done;
                        if (!issue_s(kv_it + 1, j + 2 == n)) goto done;
                    }
                }
            }
        } else if (warp == 18 && lane == 0) {
            const uint64_t kn_desc = smem_desc(smem_u32(sm.k[0]), DqSmem::CHUNK, 1024);   // N-major (dQ)
            uint32_t kv_it = 0, it_n = 0, g = 0;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it_n) {
                const int n = qtile_nkv(qts[item / hq]);
                for (int j = 0; j < n; ++j, ++kv_it, ++g) {
                    // dQ += dS K once dS is in TMEM (and, for the first tile, the last item's dQ has been read)
                    if (!bwait(&sm.ds_ready[g & 1], (g >> 1) & 1, abort_flag)) goto done;
                    if (j == 0 && !bwait(&sm.dq_free, (it_n & 1) ^ 1, abort_flag)) goto done;
                    tc_fence_after();
                    const int sk = kv_it % DQ_KSTAGES;
                    const uint64_t bk = kn_desc + uint64_t(sk) * (TB >> 4);
                    const uint32_t ads = tmem + COL_DP + 128 * (g & 1);
                    const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ts(tmem + COL_DQ, ads + 32 * (kk >> 1) + 8 * (kk & 1), desc_adv(bk, kk * 2048), ID_DQ,
                                kk > 0 ? 1u : acc0);
                    umma_commit(&sm.k_empty[sk]);
                    umma_commit(&sm.dq_done[g & 1]);
                }
                umma_commit(&sm.dq_full);
            }
        }
    } else {
        // ------------------------------------------------------------------ gradient warpgroups (warps 0-15)
        // Four warpgroups, each taking 32 key columns of every tile: more warps per scheduler hide the latency of
        // the TMEM loads (a thread's tcgen05.wait::ld waits for all of its loads, so only other warps can).
        // dP(j+1) is issued before S(j+1), so a warp may finish dS(j+1) while another is still on dS(j): ds_ready
        // alternates between two barriers by step parity so that such an early arrival never completes step j's
        // phase. Two steps ahead cannot happen: dP(j+2) waits for all of step j's arrivals.
        const int wx = warp >> 2, wl = warp & 3;
        const int rt = wl * 32 + lane;                                 // query row within the tile = TMEM lane
        const uint32_t lane_off = uint32_t(wl * 32) << 16;
        const int cb = 32 * wx;                                        // this warpgroup's key columns
        uint32_t g = 0, it_n = 0;
        const int32_t *seg_start = meta_ptr<int32_t>(meta, hd.off_seg_start);
        // Item epilogue, run after the next item's first P (so S and dP of the next tiles keep the tensor pipe
        // busy): dQ rows in bf16 (dS carried the scale); warpgroup x writes head dims [32x, 32x+32). The
        // accumulator is released as soon as it is in registers.
        bool ep_in = false;
        __nv_bfloat16 *ep_dst = dQ;
        auto epilogue = [&](uint32_t en) -> bool {
            if (!bwait(&sm.dq_full, en & 1, abort_flag)) return false;
            tc_fence_after();
            uint32_t a0[32];
            tmem_ld32(tmem + lane_off + COL_DQ + cb, a0);
            tmem_wait_ld(a0);
            tc_fence_before();
            mbar_arrive(&sm.dq_free);
            if (ep_in) {
                uint4 *dst = reinterpret_cast<uint4 *>(ep_dst);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_uint4(pack_bf16x2(__uint_as_float(a0[8 * e]), __uint_as_float(a0[8 * e + 1])),
                                        pack_bf16x2(__uint_as_float(a0[8 * e + 2]), __uint_as_float(a0[8 * e + 3])),
                                        pack_bf16x2(__uint_as_float(a0[8 * e + 4]), __uint_as_float(a0[8 * e + 5])),
                                        pack_bf16x2(__uint_as_float(a0[8 * e + 6]), __uint_as_float(a0[8 * e + 7])));
            }
            return true;
        };
        // The next item's tile is loaded at the start of this one and its per-row values (segment start, -lse/scale,
        // -D) after this item's first P, so no global load latency sits on the first step of an item.
        const QTile *qts = meta_ptr<QTile>(meta, hd.off_qts);
        auto row_values = [&](const QTile &t, int item, int &s0, float2 &lv) {
            const int row = t.row0 + rt;
            s0 = row < t.gstart + t.glen ? seg_start[row] : 0;
            lv = ldg[int64_t(item % hq) * rows_pad + row];            // padded past T
        };
        QTile tn{};
        int s0n = 0;
        float2 lvn = make_float2(0.f, 0.f);
        if (blockIdx.x < n_items) {
            tn = qts[blockIdx.x / hq];
            row_values(tn, blockIdx.x, s0n, lvn);
        }
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it_n) {
            DqItem w;
            w.t = tn;
            w.h = item % hq;
            const int nxt = item + gridDim.x;
            if (nxt < n_items) tn = qts[nxt / hq];
            const int n = qtile_nkv(w.t);
            const int row = w.t.row0 + rt;
            const bool in_group = row < w.t.gstart + w.t.glen;
            const int s0 = s0n;
            const int pfx_end = w.t.gstart + w.t.plen;
            const int x0 = w.t.row0 - w.t.gstart;
            const float2 lv = lvn;                                     // (-lse / scale, -D)
            const float c0 = lv.x * sl2;                               // - lse * log2 e
            for (int j = 0; j < n; ++j, ++g) {
                const int yt = qtile_kv(w.t, j) * FWD_BN;
                const int y0 = w.t.gstart + yt + cb;                   // first key of this warpgroup's columns
                const int cls = tile_class(x0, FWD_BM, yt, FWD_BN, w.t.glen, w.t.plen, w.t.s0first, w.t.s0last);
                const int lim_diag = in_group ? row - y0 : -1;         // allowed: c <= lim_diag and
                const int lim_pfx = pfx_end - y0;                      //   (c < lim_pfx or c >= lim_seg)
                const int lim_seg = s0 - y0;
                // P = exp2(S scale log2 e - lse log2 e), packed bf16, kept for the dS step
                if (!bwait(&sm.s_full, g & 1, abort_flag)) goto done;
                tc_fence_after();
                uint32_t pk[16];
                {
                    uint32_t a0[32];
                    tmem_ld32(tmem + lane_off + COL_S + cb, a0);
                    tmem_wait_ld(a0);
                    tc_fence_before();
                    mbar_arrive(&sm.s_free);
                    const float2 sl2v = make_float2(sl2, sl2), c0v = make_float2(c0, c0);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int c = 2 * e;
                        const float2 x = ffma2(make_float2(__uint_as_float(a0[c]), __uint_as_float(a0[c + 1])), sl2v,
                                               c0v);
                        float p0, p1;
                        if (e % DQ_POLY_EVERY == DQ_POLY_EVERY - 1) {       // this pair on the FMA pipe
                            const float2 pp = ex2_poly2(x);
                            p0 = pp.x;
                            p1 = pp.y;
                        } else {
                            p0 = ex2_approx(x.x);
                            p1 = ex2_approx(x.y);
                        }
                        if (cls != TILE_FULL) {
                            if (!(c <= lim_diag && (c < lim_pfx || c >= lim_seg))) p0 = 0.f;
                            if (!(c + 1 <= lim_diag && (c + 1 < lim_pfx || c + 1 >= lim_seg))) p1 = 0.f;
                        }
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                }
                if (j == 0) {
                    if (it_n > 0 && !epilogue(it_n - 1)) goto done;
                    ep_in = in_group;
                    ep_dst = dQ + (int64_t(row) * hq + w.h) * 128 + cb;
                    if (nxt < n_items) row_values(tn, nxt, s0n, lvn);
                }
                // dS = scale P (dP - D) -> this step's dP buffer, TMEM columns [cb, cb+16) (already read)
                const uint32_t cdp = COL_DP + 128 * (g & 1);
                if (!bwait(&sm.dp_full[g & 1], (g >> 1) & 1, abort_flag)) goto done;
                tc_fence_after();
                {
                    uint32_t a0[32];
                    tmem_ld32(tmem + lane_off + cdp + cb, a0);
                    tmem_wait_ld(a0);
                    uint32_t d0[16];
                    const float2 dv = make_float2(lv.y, lv.y), sc = make_float2(scale, scale);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint32_t p = pk[e];
                        const float2 ps = fmul2(make_float2(bf16lo(p), bf16hi(p)), sc);
                        const float2 dp = fadd2(make_float2(__uint_as_float(a0[2 * e]), __uint_as_float(a0[2 * e + 1])),
                                                dv);
                        const float2 ds = fmul2(ps, dp);
                        d0[e] = pack_bf16x2(ds.x, ds.y);
                    }
                    tmem_st16(tmem + lane_off + cdp + cb, d0);
                    tmem_wait_st();
                }
                tc_fence_before();
                mbar_arrive(&sm.ds_ready[g & 1]);
            }
        }
        if (it_n > 0 && !epilogue(it_n - 1)) goto done;
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 17) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------------------------------
// dQ from kept dS tiles. When the workspace holds a dS tile per backward step (the key-side kernel wrote each step's
// dS^T, [128 key rows][128 query columns] bf16, with scale folded in), dQ needs no recomputation:
//   dQ(query tile, q head) = sum over its key tiles of dS K      (M = 128 queries, N = d, K = 128 keys)
// A work item is (query tile, q head) in the forward's cost order. Per key tile one dS tile and one K tile come in
// through a 3-stage TMA ring; dS is the MMA's A operand read M-major (queries run along the tile's rows), K its B
// operand read N-major. dQ accumulates in one of two TMEM buffers, so the epilogue of an item overlaps the next
// item's MMAs. The kernel streams the dS tiles once: it is bound by their HBM read.
constexpr int DQS_STAGES = 3;
constexpr int DQS_THREADS = 192;     // warps 0-3 epilogue (TMEM lanes 0-127), warp 4 TMA, warp 5 TMEM + MMA issue

struct DqsSmem {
    static constexpr int TILE = 128 * 128 * 2;
    static constexpr int CHUNK = 128 * 64 * 2;
    alignas(1024) uint8_t ds[DQS_STAGES][TILE];
    alignas(1024) uint8_t k[DQS_STAGES][TILE];
    uint64_t full[DQS_STAGES], empty[DQS_STAGES], acc_full[2], acc_empty[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(DqsSmem) + 1024 <= 232448, "dQ (kept dS) kernel shared memory exceeds 227 KB");

// tmDS: 3-D map over the dS slots viewed as [slots * 128 rows][1][128 columns], box (64, 1, 128).
__global__ void __launch_bounds__(DQS_THREADS, 1)
k_bwd_dq_ds(const __grid_constant__ CUtensorMap tmDS, const __grid_constant__ CUtensorMap tmK,
            const void *__restrict__ meta, __nv_bfloat16 *__restrict__ dQ, int hq, int hkv, const void *ds_buf,
            int64_t ds_cap) {
    extern __shared__ uint8_t smem_raw[];
    DqsSmem &sm = *reinterpret_cast<DqsSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
    if (hd.dev_err != 0 || ds_buf == nullptr || int64_t(hd.n_slots) * hkv > ds_cap) return;   // k_bwd_dq does dQ
    const int r = hq / hkv;
    const int n_items = hd.n_qt * hq;
    const int32_t *kslot = meta_ptr<int32_t>(meta, hd.off_kslot);
    const int32_t *kfirst = meta_ptr<int32_t>(meta, hd.off_kfirst);
    volatile int *abort_flag = &sm.abort_flag;
    if (threadIdx.x == 0) {
        for (int s = 0; s < DQS_STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.acc_full[b], 1);
            mbar_init(&sm.acc_empty[b], 128);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&sm.tmem_base, 256);
        tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        prefetch_tmap(&tmDS);
        prefetch_tmap(&tmK);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t u = 0;
            for (int rnd = 0, item = blockIdx.x; item < n_items; item = alt_item(++rnd, blockIdx.x, gridDim.x)) {
                const DqItem w = dq_decode(meta, hd, item, hq, hkv);
                const int n = qtile_nkv(w.t);
                const int qt = (w.t.row0 - w.t.gstart) / BWD_BM;       // query tile within the group
                const int k0 = kfirst[w.t.group];
                for (int j = 0; j < n; ++j, ++u) {
                    const int kl = qtile_kv(w.t, j);                    // key tile within the group (= its first
                    const int64_t slot = int64_t(w.kh) * hd.n_slots + kslot[k0 + kl] + int64_t(qt - kl) * r +
                                         (w.h - w.kh * r);
                    const int st = u % DQS_STAGES;                     //  attending query tile)
                    if (!bwait(&sm.empty[st], ((u / DQS_STAGES) & 1) ^ 1, abort_flag)) goto done;
                    mbar_arrive_expect_tx(&sm.full[st], 2 * DqsSmem::TILE);
                    for (int c = 0; c < 2; ++c) {
                        tma_load_3d(sm.ds[st] + c * DqsSmem::CHUNK, &tmDS, c * 64, 0, int32_t(slot * BWD_BN),
                                    &sm.full[st]);
                        tma_load_3d(sm.k[st] + c * DqsSmem::CHUNK, &tmK, c * 64, w.kh, w.t.gstart + kl * BWD_BN,
                                    &sm.full[st]);
                    }
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t ID = idesc_bf16(128, 128, 1, 1);        // A = dS (M-major), B = K (N-major)
            const uint64_t a_desc = smem_desc(smem_u32(sm.ds[0]), DqsSmem::CHUNK, 1024);
            const uint64_t b_desc = smem_desc(smem_u32(sm.k[0]), DqsSmem::CHUNK, 1024);
            uint32_t u = 0, it_n = 0;
            for (int rnd = 0, item = blockIdx.x; item < n_items; item = alt_item(++rnd, blockIdx.x, gridDim.x), ++it_n) {
                const int n = qtile_nkv(meta_ptr<QTile>(meta, hd.off_qts)[item / hq]);
                const uint32_t b = it_n & 1;
                if (!bwait(&sm.acc_empty[b], ((it_n >> 1) & 1) ^ 1, abort_flag)) goto done;
                for (int j = 0; j < n; ++j, ++u) {
                    const int st = u % DQS_STAGES;
                    if (!bwait(&sm.full[st], (u / DQS_STAGES) & 1, abort_flag)) goto done;
                    tc_fence_after();
                    const uint64_t a = a_desc + uint64_t(st) * (DqsSmem::TILE >> 4);
                    const uint64_t bb = b_desc + uint64_t(st) * (DqsSmem::TILE >> 4);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ss(tmem + 128 * b, desc_adv(a, kk * 2048), desc_adv(bb, kk * 2048), ID,
                                (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sm.empty[st]);
                }
                umma_commit(&sm.acc_full[b]);
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue warps (thread = query row)
        const uint32_t lane_off = uint32_t(warp * 32) << 16;
        const int rt = warp * 32 + lane;
        const bool dq_v8 = aligned32(dQ);                                // rows are 256 bytes: the base decides
        uint32_t it_n = 0;
        for (int rnd = 0, item = blockIdx.x; item < n_items; item = alt_item(++rnd, blockIdx.x, gridDim.x), ++it_n) {
            const DqItem w = dq_decode(meta, hd, item, hq, hkv);
            const uint32_t b = it_n & 1;
            const int row = w.t.row0 + rt;
            const bool in_group = row < w.t.gstart + w.t.glen;
            if (!bwait(&sm.acc_full[b], (it_n >> 1) & 1, abort_flag)) goto done;
            tc_fence_after();
            uint32_t a[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_off + 128 * b + 32 * c, a[c]);
            tmem_wait_ld(a[0], a[1], a[2], a[3]);
            tc_fence_before();
            mbar_arrive(&sm.acc_empty[b]);
            if (in_group) {                                            // 256 bytes: eight 32-byte stores
                __nv_bfloat16 *dst = dQ + (int64_t(row) * hq + w.h) * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const uint32_t *x = a[c] + 16 * e;
                        st_global_32(dst + 32 * c + 16 * e, dq_v8, pack_bf16x2(__uint_as_float(x[0]), __uint_as_float(x[1])),
                                     pack_bf16x2(__uint_as_float(x[2]), __uint_as_float(x[3])),
                                     pack_bf16x2(__uint_as_float(x[4]), __uint_as_float(x[5])),
                                     pack_bf16x2(__uint_as_float(x[6]), __uint_as_float(x[7])),
                                     pack_bf16x2(__uint_as_float(x[8]), __uint_as_float(x[9])),
                                     pack_bf16x2(__uint_as_float(x[10]), __uint_as_float(x[11])),
                                     pack_bf16x2(__uint_as_float(x[12]), __uint_as_float(x[13])),
                                     pack_bf16x2(__uint_as_float(x[14]), __uint_as_float(x[15])));
                    }
            }
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace pp
