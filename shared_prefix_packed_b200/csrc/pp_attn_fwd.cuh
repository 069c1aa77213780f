// pp_attn_fwd.cuh - forward of exact attention over a preference-packed sequence.
//
// What it computes (pp.h, pp_attn_fwd): per q head h (kv head h / r), s_ij = scale q_i.k_j over the allowed keys
// of row i, lse_i = ln sum_j exp(s_ij), o_i = sum_j exp(s_ij - lse_i) v_j. The allowed set (pp_meta.cuh) is the
// prefix/own-response mask the pages imply ("Preference Packing" method digest; "prefix_grouper_utils.py" diagram).
//
// Tensor-core kernel (bf16, sm_100a). One persistent CTA per SM walks work items (query tile of 128 rows, GQA pair
// of q heads sharing one kv head) in cost order. Warp roles:
//   warps 0-3  softmax for head slot 0 (TMEM lanes 0-127 = the tile's rows)
//   warps 4-7  softmax for head slot 1
//   warp 8     TMA producer: Q of both heads once per item, then K (3-stage ring, one tile ahead) and V (2 stages)
//   warp 9     TMEM allocator and the single MMA-issuing thread
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 [384,384+d); P_h (bf16) overwrites the first
// 64 columns of S_h once the softmax has read S_h. Per key tile the MMA thread issues, ping-ponging the heads,
//   PV0(j) -> S0(j+1) -> PV1(j) -> S1(j+1)
// so the tensor cores work on one head while the other head's softmax runs. MMAs from one thread execute in
// issue order, which makes S_h(j+1) safe to issue right after PV_h(j), the MMA that reads P_h(j).
// Only the key tiles the schedule lists are visited ("PackInfer" abstract: attention directly over the packed
// query-key regions); sibling-response tiles are never loaded. FULL tiles skip the element mask.
// Softmax: exp2 with the scale folded in; the running max is only raised when a tile's max exceeds it by more than
// 8 (log2 units), so the O rescale (a TMEM round trip) is rare; the result is exact up to rounding either way. One
// pair of exponentials in FWD_POLY_EVERY is computed on the FMA pipe (ex2_poly2) instead of the MUFU unit, whose 16
// results per clock per SM would otherwise take as long as the tile's MMAs.
#pragma once
#include <cuda_bf16.h>
#include "pp_meta.cuh"
#include "pp_ptx.cuh"
#include "pp_build.cuh"   // g_dev_err, DEVERR_*

namespace pp {

constexpr int FWD_THREADS = 320;
constexpr int FWD_KSTAGES = 3;   // K is needed one step earlier than V (S(j+1) is issued right after PV(j))
constexpr int FWD_VSTAGES = 2;
constexpr int FWD_POLY_EVERY = 4; // one pair in four exponentials goes to the FMA pipe (ex2_poly2)
constexpr float FWD_RESCALE_THRESHOLD = 8.0f;
constexpr uint64_t WAIT_TIMEOUT_NS = 2000000000ull;   // bounded waits: 2 s, then the kernel reports and leaves

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded mbarrier wait. On timeout (limit_ns) it records DEVERR_TIMEOUT, raises the CTA's abort flag and returns
// false; every other waiter of the CTA then gives up at its next poll.
__device__ __forceinline__ bool bwait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                      uint64_t limit_ns = WAIT_TIMEOUT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
        if ((it & 7) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicOr(&g_dev_err, DEVERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Self-test of the bounded wait: one CTA waits, with the kernels' own bwait and the given limit, on an mbarrier that
// nothing ever arrives on. It issues no copy and no MMA, so nothing is in flight when the wait gives up; the
// timeout is reported through the device error word like any other. waited_ns receives the time the wait took.
__global__ void k_selftest_wait(uint64_t limit_ns, unsigned long long *waited_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = globaltimer_ns();
        const bool ok = bwait(&bar, 0, &abort_flag, limit_ns);
        *waited_ns = ok ? 0ull : static_cast<unsigned long long>(globaltimer_ns() - t0);
    }
}

template <int D>
struct FwdSmem {
    static constexpr int TILE_BYTES = 128 * D * 2;      // one 128-row tile of bf16 [rows][D]
    static constexpr int CHUNK_BYTES = 128 * 64 * 2;    // one 64-column swizzled chunk of such a tile
    alignas(1024) uint8_t q[2][TILE_BYTES];
    alignas(1024) uint8_t k[FWD_KSTAGES][TILE_BYTES];
    alignas(1024) uint8_t v[FWD_VSTAGES][TILE_BYTES];
    uint64_t q_full, q_empty;
    uint64_t k_full[FWD_KSTAGES], k_empty[FWD_KSTAGES], v_full[FWD_VSTAGES], v_empty[FWD_VSTAGES];
    uint64_t s_full[2], p_full[2], o_done[2], o_free[2];
    uint32_t tmem_base;
    int abort_flag;
};

static_assert(sizeof(FwdSmem<128>) + 1024 <= 232448, "forward shared memory exceeds 227 KB");

struct FwdItem {
    QTile t;
    int h0, nh, kh;
};

__device__ __forceinline__ FwdItem fwd_decode(const void *meta, const MetaHeader &hd, int item, int hq, int hkv) {
    const int r = hq / hkv;
    const int spk = (r + 1) / 2;              // head pairs per kv head
    const int nslots = hkv * spk;
    const int qi = item / nslots, slot = item % nslots;
    FwdItem it;
    it.kh = slot / spk;
    const int pr = slot % spk;
    it.h0 = it.kh * r + 2 * pr;
    it.nh = (2 * pr + 1 < r) ? 2 : 1;
    it.t = meta_ptr<QTile>(meta, hd.off_qts)[qi];
    return it;
}

template <int D>
__global__ void __launch_bounds__(FWD_THREADS, 1)
k_attn_fwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const void *__restrict__ meta,
              __nv_bfloat16 *__restrict__ O, float *__restrict__ LSE, int hq, int hkv, float sl2) {
    extern __shared__ uint8_t smem_raw[];
    FwdSmem<D> &sm = *reinterpret_cast<FwdSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                      ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
    const int T = hd.T;
    const int r = hq / hkv;
    const int n_items = hd.n_qt * hkv * ((r + 1) / 2);
    const int32_t *seg_start = meta_ptr<int32_t>(meta, hd.off_seg_start);
    volatile int *abort_flag = &sm.abort_flag;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, 1);
        for (int s = 0; s < FWD_KSTAGES; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int s = 0; s < FWD_VSTAGES; ++s) {
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&sm.s_full[h], 1);
            mbar_init(&sm.o_done[h], 1);
            mbar_init(&sm.p_full[h], 128);
            mbar_init(&sm.o_free[h], 128);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (hd.dev_err == 0 && warp == 8 && lane == 0) {
        // ------------------------------------------------------------------ TMA producer
        uint32_t kv_it = 0, n_it = 0;
        for (int rnd = 0, item = blockIdx.x; item < n_items; item = alt_item(++rnd, blockIdx.x, gridDim.x)) {
            const FwdItem w = fwd_decode(meta, hd, item, hq, hkv);
            const int n = qtile_nkv(w.t);
            const int nxt = alt_item(rnd + 1, blockIdx.x, gridDim.x);
            if (nxt < n_items) {                                       // the next item's Q into L2 (read once, so
                const FwdItem wn = fwd_decode(meta, hd, nxt, hq, hkv);  // a miss otherwise)
                for (int hs = 0; hs < wn.nh; ++hs)
                    for (int c = 0; c < D / 64; ++c) tma_prefetch_3d(&tmQ, c * 64, wn.h0 + hs, wn.t.row0);
            }
            if (!bwait(&sm.q_empty, (n_it & 1) ^ 1, abort_flag)) goto done;
            ++n_it;
            mbar_arrive_expect_tx(&sm.q_full, w.nh * FwdSmem<D>::TILE_BYTES);
            for (int hs = 0; hs < w.nh; ++hs)
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sm.q[hs] + c * FwdSmem<D>::CHUNK_BYTES, &tmQ, c * 64, w.h0 + hs, w.t.row0,
                                &sm.q_full);
            // K runs one tile ahead of V: K(j + 1) is issued before V(j), since S(j + 1) follows PV(j) directly
            auto load_k = [&](uint32_t it, int jj) -> bool {
                const int s = it % FWD_KSTAGES;
                if (!bwait(&sm.k_empty[s], ((it / FWD_KSTAGES) & 1) ^ 1, abort_flag)) return false;
                mbar_arrive_expect_tx(&sm.k_full[s], FwdSmem<D>::TILE_BYTES);
                const int y0 = w.t.gstart + qtile_kv(w.t, jj) * FWD_BN;
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sm.k[s] + c * FwdSmem<D>::CHUNK_BYTES, &tmK, c * 64, w.kh, y0, &sm.k_full[s]);
                return true;
            };
            if (n > 0 && !load_k(kv_it, 0)) goto done;
            for (int j = 0; j < n; ++j, ++kv_it) {
                if (j + 1 < n && !load_k(kv_it + 1, j + 1)) goto done;
                const int y0 = w.t.gstart + qtile_kv(w.t, j) * FWD_BN;
                const int s = kv_it % FWD_VSTAGES;
                if (!bwait(&sm.v_empty[s], ((kv_it / FWD_VSTAGES) & 1) ^ 1, abort_flag)) goto done;
                mbar_arrive_expect_tx(&sm.v_full[s], FwdSmem<D>::TILE_BYTES);
                for (int c = 0; c < D / 64; ++c)
                    tma_load_3d(sm.v[s] + c * FwdSmem<D>::CHUNK_BYTES, &tmV, c * 64, w.kh, y0, &sm.v_full[s]);
            }
        }
    } else if (hd.dev_err == 0 && warp == 9 && lane == 0) {
        // ------------------------------------------------------------------ MMA issuer
        constexpr uint32_t IDESC_S = idesc_bf16(128, FWD_BN, 0, 0);
        constexpr uint32_t IDESC_O = idesc_bf16(128, D, 0, 1);
        uint32_t kv_it = 0, n_it = 0, p_cnt[2] = {0, 0}, item_cnt[2] = {0, 0};
        // descriptors built once; a head slot or stage is a constant stride away (desc_adv)
        constexpr uint32_t TB = FwdSmem<D>::TILE_BYTES;
        const uint64_t q_desc = smem_desc(smem_u32(sm.q[0]), 16, 1024);
        const uint64_t k_desc = smem_desc(smem_u32(sm.k[0]), 16, 1024);
        const uint64_t v_desc = smem_desc(smem_u32(sm.v[0]), FwdSmem<D>::CHUNK_BYTES, 1024);
        auto issue_s = [&](int hs, int st) {
            const uint64_t a = q_desc + uint64_t(hs) * (TB >> 4), b = k_desc + uint64_t(st) * (TB >> 4);
            const uint32_t d = tmem + hs * 128;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * FwdSmem<D>::CHUNK_BYTES + (kk & 3) * 32;
                umma_ss(d, desc_adv(a, off), desc_adv(b, off), IDESC_S, kk > 0);
            }
        };
        auto issue_pv = [&](int hs, int st, uint32_t acc) {
            const uint64_t b = v_desc + uint64_t(st) * (TB >> 4);
            const uint32_t d = tmem + 256 + hs * 128, a = tmem + hs * 128;
#pragma unroll
            for (int kk = 0; kk < FWD_BN / 16; ++kk)
                umma_ts(d, a + kk * 8, desc_adv(b, kk * 2048), IDESC_O, (acc | kk) ? 1u : 0u);
        };
        for (int rnd = 0, item = blockIdx.x; item < n_items; item = alt_item(++rnd, blockIdx.x, gridDim.x)) {
            const FwdItem w = fwd_decode(meta, hd, item, hq, hkv);
            const int n = qtile_nkv(w.t);
            if (!bwait(&sm.q_full, n_it & 1, abort_flag)) goto done;
            ++n_it;
            int st = kv_it % FWD_KSTAGES;
            if (!bwait(&sm.k_full[st], (kv_it / FWD_KSTAGES) & 1, abort_flag)) goto done;
            tc_fence_after();
            for (int hs = 0; hs < w.nh; ++hs) {
                issue_s(hs, st);
                umma_commit(&sm.s_full[hs]);
            }
            umma_commit(&sm.k_empty[st]);
            for (int j = 0; j < n; ++j) {
                st = (kv_it + j) % FWD_VSTAGES;
                const int st2 = (kv_it + j + 1) % FWD_KSTAGES;
                if (!bwait(&sm.v_full[st], ((kv_it + j) / FWD_VSTAGES) & 1, abort_flag)) goto done;
                bool have_next = j + 1 < n;
                if (have_next && !bwait(&sm.k_full[st2], ((kv_it + j + 1) / FWD_KSTAGES) & 1, abort_flag)) goto done;
                for (int hs = 0; hs < w.nh; ++hs) {
                    if (j == 0 && !bwait(&sm.o_free[hs], (item_cnt[hs] & 1) ^ 1, abort_flag)) goto done;
                    if (!bwait(&sm.p_full[hs], p_cnt[hs] & 1, abort_flag)) goto done;
                    ++p_cnt[hs];
                    tc_fence_after();
                    issue_pv(hs, st, j > 0 ? 1u : 0u);
                    umma_commit(&sm.o_done[hs]);
                    if (have_next) {
                        issue_s(hs, st2);
                        umma_commit(&sm.s_full[hs]);
                    }
                }
                umma_commit(&sm.v_empty[st]);
                if (have_next) umma_commit(&sm.k_empty[st2]);
            }
            umma_commit(&sm.q_empty);
            kv_it += n;
            for (int hs = 0; hs < w.nh; ++hs) ++item_cnt[hs];
        }
    } else if (hd.dev_err == 0 && warp < 8) {
        // ------------------------------------------------------------------ softmax warpgroups
        const int wg = warp >> 2;
        const int lane_base = (warp & 3) * 32;
        const int rt = lane_base + lane;                       // row within the tile = TMEM lane
        const uint32_t t_s = tmem + (uint32_t(lane_base) << 16) + wg * 128;
        const uint32_t t_o = tmem + (uint32_t(lane_base) << 16) + 256 + wg * 128;
        const bool o_v8 = aligned32(O);                                  // rows are d * 2 bytes: the base decides
        uint32_t s_cnt = 0, pv_cnt = 0;
        for (int rnd = 0, item = blockIdx.x; item < n_items; item = alt_item(++rnd, blockIdx.x, gridDim.x)) {
            const FwdItem w = fwd_decode(meta, hd, item, hq, hkv);
            if (wg >= w.nh) continue;
            const int h = w.h0 + wg;
            const int n = qtile_nkv(w.t);
            const int row = w.t.row0 + rt;
            const int gend = w.t.gstart + w.t.glen;
            const bool in_group = row < gend;
            const int s0 = in_group ? seg_start[row] : 0;
            const int pfx_end = w.t.gstart + w.t.plen;
            const int x0 = w.t.row0 - w.t.gstart;
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < n; ++j) {
                const int yt = qtile_kv(w.t, j) * FWD_BN;
                const int y0 = w.t.gstart + yt;
                const int cls = tile_class(x0, FWD_BM, yt, FWD_BN, w.t.glen, w.t.plen, w.t.s0first, w.t.s0last);
                if (!bwait(&sm.s_full[wg], s_cnt & 1, abort_flag)) goto done;
                ++s_cnt;
                tc_fence_after();
                float s[FWD_BN];
                {   // all four loads in flight before one wait
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    tmem_ld32(t_s, r0);
                    tmem_ld32(t_s + 32, r1);
                    tmem_ld32(t_s + 64, r2);
                    tmem_ld32(t_s + 96, r3);
                    tmem_wait_ld(r0, r1, r2, r3);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        s[e] = __uint_as_float(r0[e]);
                        s[32 + e] = __uint_as_float(r1[e]);
                        s[64 + e] = __uint_as_float(r2[e]);
                        s[96 + e] = __uint_as_float(r3[e]);
                    }
                }
                if (cls != TILE_FULL) {
                    // allowed iff y <= row, and y in the prefix or in row's own segment; nothing for rows outside
                    const int lim_diag = in_group ? row - y0 : -1;
                    const int lim_pfx = pfx_end - y0;
                    const int lim_seg = s0 - y0;
#pragma unroll
                    for (int c = 0; c < FWD_BN; ++c)
                        if (!(c <= lim_diag && (c < lim_pfx || c >= lim_seg))) s[c] = -INFINITY;
                }
                float m4[4] = {s[0], s[1], s[2], s[3]};                 // four independent max chains
#pragma unroll
                for (int c = 4; c < FWD_BN; c += 2) m4[(c >> 1) & 3] = fmax3(m4[(c >> 1) & 3], s[c], s[c + 1]);
                const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                const float mt = mx * sl2;
                bool rescale = false;
                float alpha = 1.f;
                if (mt > m + FWD_RESCALE_THRESHOLD) {
                    if (j > 0 && m != -INFINITY) {
                        rescale = true;
                        alpha = ex2_approx(m - mt);
                    }
                    l *= alpha;
                    m = mt;
                }
                const float mu = (m == -INFINITY) ? 0.f : m;
                // scale/shift and row sum on packed fp32 pairs (one instruction per pair)
                float2 ls[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // two independent pair chains
                const float2 sl2v = make_float2(sl2, sl2), nmu = make_float2(-mu, -mu);
#pragma unroll
                for (int c = 0; c < FWD_BN / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 x = ffma2(make_float2(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]), sl2v, nmu);
                        float p0, p1;
                        if (e % FWD_POLY_EVERY == FWD_POLY_EVERY - 1) {     // this pair on the FMA pipe
                            const float2 pp = ex2_poly2(x);
                            p0 = pp.x;
                            p1 = pp.y;
                        } else {
                            p0 = ex2_approx(x.x);
                            p1 = ex2_approx(x.y);
                        }
                        ls[e & 1] = fadd2(ls[e & 1], make_float2(p0, p1));
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(t_s + c * 16, pk);
                }
                l += (ls[0].x + ls[0].y) + (ls[1].x + ls[1].y);
                tmem_wait_st();
                // tcgen05.ld/st are warp-collective: the whole warp takes the rescale path if any row needs it
                if (__any_sync(0xffffffffu, rescale)) {
                    // O holds the sum over earlier tiles at the old max: wait for PV(j-1), then scale it
                    if (!bwait(&sm.o_done[wg], (pv_cnt + j - 1) & 1, abort_flag)) goto done;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t rr[32];
                        tmem_ld32(t_o + c * 32, rr);
                        tmem_wait_ld(rr);
#pragma unroll
                        for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
                        tmem_st32(t_o + c * 32, rr);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                mbar_arrive(&sm.p_full[wg]);
            }
            // epilogue: O / l, LSE
            if (!bwait(&sm.o_done[wg], (pv_cnt + n - 1) & 1, abort_flag)) goto done;
            pv_cnt += n;
            tc_fence_after();
            {
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                __nv_bfloat16 *orow = O + (int64_t(row) * hq + h) * D;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(t_o + c * 32, rr);
                    tmem_wait_ld(rr);
                    if (in_group) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            pk[e] = pack_bf16x2(__uint_as_float(rr[2 * e]) * inv_l,
                                                __uint_as_float(rr[2 * e + 1]) * inv_l);
#pragma unroll
                        for (int e = 0; e < 2; ++e)                        // 64 bytes: two 32-byte stores
                            st_global_32(orow + c * 32 + 16 * e, o_v8, pk[8 * e], pk[8 * e + 1], pk[8 * e + 2], pk[8 * e + 3],
                                         pk[8 * e + 4], pk[8 * e + 5], pk[8 * e + 6], pk[8 * e + 7]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.o_free[wg]);
            if (in_group) LSE[int64_t(h) * T + row] = (m + __log2f(l)) * 0.69314718055994531f;
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------------------------------
// fp32 CUDA-core forward (PP_FP32). Same schedule and mask; one block per (query tile, q head), one thread per row,
// K/V tiles staged in shared memory, fp32 accumulation with an exact (per key) online softmax.
template <typename T, int D>
__global__ void __launch_bounds__(128) k_attn_fwd_simt(const T *__restrict__ q, const T *__restrict__ k,
                                                       const T *__restrict__ v, const void *__restrict__ meta,
                                                       T *__restrict__ o, float *__restrict__ lse, int hq, int hkv,
                                                       float scale) {
    extern __shared__ float sf[];
    float *sK = sf;
    float *sV = sf + FWD_BN * D;
    const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
    if (hd.dev_err) return;
    const int Tn = hd.T;
    const int r = hq / hkv;
    const QTile *qts = meta_ptr<QTile>(meta, hd.off_qts);
    const int32_t *seg_start = meta_ptr<int32_t>(meta, hd.off_seg_start);
    const int n_items = hd.n_qt * hq;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const QTile t = qts[item / hq];
        const int h = item % hq, kh = h / r;
        const int row = t.row0 + threadIdx.x;
        const bool in_group = row < t.gstart + t.glen;
        const int s0 = in_group ? seg_start[row] : 0;
        const int pfx_end = t.gstart + t.plen;
        float qv[D], acc[D];
#pragma unroll
        for (int e = 0; e < D; ++e) {
            qv[e] = in_group ? static_cast<float>(q[(int64_t(row) * hq + h) * D + e]) : 0.f;
            acc[e] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        const int n = qtile_nkv(t);
        for (int j = 0; j < n; ++j) {
            const int y0 = t.gstart + qtile_kv(t, j) * FWD_BN;
            __syncthreads();
            for (int e = threadIdx.x; e < FWD_BN * D; e += blockDim.x) {
                const int c = e / D, dd = e % D;
                const int y = y0 + c;
                sK[e] = y < Tn ? static_cast<float>(k[(int64_t(y) * hkv + kh) * D + dd]) : 0.f;
                sV[e] = y < Tn ? static_cast<float>(v[(int64_t(y) * hkv + kh) * D + dd]) : 0.f;
            }
            __syncthreads();
            if (!in_group) continue;
            for (int c = 0; c < FWD_BN; ++c) {
                const int y = y0 + c;
                if (!(y <= row && (y < pfx_end || y >= s0))) continue;
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < D; ++e) dot = fmaf(qv[e], sK[c * D + e], dot);
                const float sc = dot * scale;
                if (sc > m) {
                    const float corr = expf(m - sc);
                    l *= corr;
#pragma unroll
                    for (int e = 0; e < D; ++e) acc[e] *= corr;
                    m = sc;
                }
                const float p = expf(sc - m);
                l += p;
#pragma unroll
                for (int e = 0; e < D; ++e) acc[e] = fmaf(p, sV[c * D + e], acc[e]);
            }
        }
        if (in_group) {
            const float inv = 1.f / l;
#pragma unroll
            for (int e = 0; e < D; ++e) o[(int64_t(row) * hq + h) * D + e] = static_cast<T>(acc[e] * inv);
            lse[int64_t(h) * Tn + row] = m + logf(l);
        }
    }
}

}  // namespace pp
