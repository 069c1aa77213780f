// pp_attn_bwd.cuh - backward of exact attention over a preference-packed sequence (bf16, d = 128, sm_100a).
//
// What it computes (pp.h, pp_attn_bwd): with p_ij = exp(s_ij - lse_i) and D_i = dO_i . o_i,
//   dS_ij = p_ij (dO_i . v_j - D_i),  dQ_i = scale sum_j dS_ij k_j,
//   dK_j = scale sum_h sum_i dS_ij q_i,  dV_j = sum_h sum_i p_ij dO_i   (h over the q heads of j's kv head).
//
// Kernels:
//   k_bwd_pre     (-lse / scale, -D) per row and head, D = rowsum(dO * O) in fp32 (HBM-bound).
//   k_bwd_tc      dK and dV: key/value-stationary tensor-core kernel (below); when the workspace has room it also
//                 keeps every step's dS^T tile there.
//   k_bwd_dq_ds   dQ = sum dS K from the kept tiles (pp_attn_bwd_dq.cuh), streaming them once.
//   k_bwd_dq      dQ when the tiles are not kept: query-stationary tensor-core kernel (pp_attn_bwd_dq.cuh) that
//                 recomputes S and dP per tile. Either way every dQ row is produced by exactly one CTA (no fp32
//                 accumulator, no reduction traffic).
//   k_bwd_convert the fp32 dK/dV partials of split key tiles to bf16.
// k_bwd_tc: a work item is (key tile of 128 rows, kv head, chunk of the query tiles that attend it). Seen from key
// y the attending queries are one interval [y, e(y)) (pp_meta.cuh), so a key tile's query tiles are one contiguous
// range; prefix key tiles (attended by every response of the group) get long ranges and are split into chunks so
// the persistent grid stays balanced. Per step (query tile of 128 rows, one q head of the kv head), four products,
// all with N = 128:
//   S^T  = K Q^T                          TMEM S
//   dP^T = V dO^T                         TMEM dP
//   gradient warps: read S^T (S^T(g+1) may then be issued), P^T = exp(S^T - lse); read dP^T; P^T (bf16) into
//                   the dP columns they have read                                          -> dV may start
//   dV  += P^T dO        (A from TMEM)    TMEM dV
//   gradient warps: dS^T = scale P^T (dP^T - D) (bf16) into the other dP columns they read  -> dK may start
//   dK  += dS^T Q        (A from TMEM)    TMEM dK
// S^T(g+1) is issued as soon as S^T(g) is in registers, so P(g+1) overlaps dV(g), dK(g) and dP^T(g+1).
// Two threads issue the MMAs: one S^T and dP^T, the other dK and dV (a thread needs about 50 cycles to issue an
// MMA, so one issuer that also polls barriers would starve the tensor pipe). dK/dV stay in TMEM for the whole item;
// an unsplit key tile writes them as bf16, a split one adds its fp32 partial into the workspace (one add per element
// and chunk).
// TMEM (512 columns): S [0,128), dP / (P^T, dS^T) [128,256), dV [256,384), dK [384,512).
// Per-query values folded into the MMAs: the gradient warps own a key row each and would otherwise need the lse
// and D of all 128 query columns per step (a shared-memory or shuffle broadcast per element, which measured
// several times slower than the exp itself). Instead one extra K = 16 slice is appended to the S^T and dP^T
// products: K and V get columns (1, 1, 1, 0, ...), Q gets (-lse/scale) and dO gets (-D), each split exactly into
// three bf16 parts (hi, mid, lo). The accumulators then hold s - lse/scale and dP - D directly, so
// P^T = exp2(S'^T * scale * log2 e) and dS^T = P^T * dP'^T * scale need nothing but the TMEM values. The extra
// slices cost 2 of 34 MMAs per step. They live in shared memory as 128 x 16 bf16 tiles in the no-swizzle
// core-matrix layout; the producer warp writes the query side for each step.
// Q/dO tiles come through 2-stage rings with separate barriers (Q is freed by dK, dO by dV), prefetched into L2 two
// steps ahead.
// Work items run in cost order within groups of four kv heads (bwd_item_split): cost order balances the static
// round-robin, and the head groups bound the Q/dO rows that concurrently running items read, so they are reused
// from L2 across key tiles. An item's epilogue (dK/dV out of TMEM) runs inside the next item's first step, between
// its P and its dS, when dK/dV of the item have long been complete.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "pp_meta.cuh"
#include "pp_ptx.cuh"
#include "pp_attn_fwd.cuh"   // bwait, globaltimer_ns
#include "pp_attn_bwd_dq.cuh"

namespace pp {

constexpr int BWD_THREADS = 352;   // 8 gradient warps, producer, two MMA issuers
constexpr int BWD_D = 128;

struct BwdWorkspace {
    int64_t rows_pad;   // T + padding rows so tiles that stick out past T stay inside the buffers
    int64_t off_delta;  // float2 [hq][rows_pad]: (-lse_i / scale, -D_i)
    int64_t off_dk;     // fp32 [rows_pad][hkv][d]: dK accumulator of split key tiles
    int64_t off_dv;     // fp32 [rows_pad][hkv][d]: dV accumulator of split key tiles
    int64_t total;
};

inline BwdWorkspace bwd_workspace_layout(int64_t T, int hq, int hkv, int d) {
    BwdWorkspace w{};
    w.rows_pad = (T + 256 + 7) & ~int64_t(7);
    int64_t o = 0;
    w.off_delta = o; o = align256(o + 8 * int64_t(hq) * w.rows_pad);
    w.off_dk = o;    o = align256(o + 4 * w.rows_pad * hkv * d);
    w.off_dv = o;    o = align256(o + 4 * w.rows_pad * hkv * d);
    w.total = o;
    return w;
}

// ------------------------------------------------------------------------------------------------- preprocess
// D = sum_d dO * O in fp32 per (row, head), stored with the lse as (-lse / scale, -D), the values the query side of
// the extra MMA slice carries; padding rows get zeros. (row, head) pairs are contiguous 256-byte rows of O and dO,
// so a warp takes eight consecutive pairs: half-warps of 16 lanes x 16 bytes, four loads of each tensor in flight
// per lane (HBM-bound). The same grid also zeroes the fp32 dK/dV accumulator rows of the split key tiles (the
// only rows the key-side kernel adds partials into); no other row of the accumulators is ever read.
__global__ void k_bwd_pre(const __nv_bfloat16 *__restrict__ O, const __nv_bfloat16 *__restrict__ dO,
                          const float *__restrict__ lse, float2 *__restrict__ ld, int64_t T, int64_t rows_pad,
                          int hq, float inv_scale, const void *__restrict__ meta, float *__restrict__ dk_acc,
                          float *__restrict__ dv_acc, int hkv) {
    {
        // zero the fp32 dK/dV rows of split key tiles (their chunks add into them). A unit is 16 rows of one key
        // tile: the rows of a tile are contiguous ([rows][hkv][d]), so a unit is one contiguous run of float4.
        const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
        if (hd.dev_err == 0 && hd.n_split > 0) {
            const KTile *kts = meta_ptr<KTile>(meta, hd.off_kt);
            const int per_row = hkv * (BWD_D / 4);                     // float4 per row
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int u = blockIdx.x; u < hd.n_kt * 8; u += gridDim.x) {
                const KTile t = kts[u >> 3];
                if (t.nch <= 1) continue;
                const int r0 = (u & 7) * 16;
                const int rows = min(16, t.gstart + t.glen - t.row0 - r0);
                if (rows <= 0) continue;
                const int64_t base = (int64_t(t.row0) + r0) * per_row;
                float4 *dk4 = reinterpret_cast<float4 *>(dk_acc) + base;
                float4 *dv4 = reinterpret_cast<float4 *>(dv_acc) + base;
                for (int e = threadIdx.x; e < rows * per_row; e += blockDim.x) {
                    dk4[e] = z;
                    dv4[e] = z;
                }
            }
        }
    }
    const int lane = threadIdx.x & 31, half = lane >> 4, hl = lane & 15;
    const int64_t n_pairs = rows_pad * hq, n_real = T * hq;
    const int64_t nwarps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t c = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); c * 8 < n_pairs; c += nwarps) {
        uint4 a[4], b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int64_t w = c * 8 + 2 * k + half;                   // pair index = row * hq + head
            if (w < n_real) {
                a[k] = reinterpret_cast<const uint4 *>(O + w * BWD_D)[hl];
                b[k] = reinterpret_cast<const uint4 *>(dO + w * BWD_D)[hl];
            } else {
                a[k] = make_uint4(0, 0, 0, 0);
                b[k] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t av[4] = {a[k].x, a[k].y, a[k].z, a[k].w}, bv[4] = {b[k].x, b[k].y, b[k].z, b[k].w};
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc = fmaf(__uint_as_float(av[e] << 16), __uint_as_float(bv[e] << 16), acc);
                acc = fmaf(__uint_as_float(av[e] & 0xffff0000u), __uint_as_float(bv[e] & 0xffff0000u), acc);
            }
#pragma unroll
            for (int off = 8; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            const int64_t w = c * 8 + 2 * k + half;
            if (hl == 0 && w < n_pairs) {
                const int64_t i = w / hq;
                const int h = static_cast<int>(w % hq);
                ld[int64_t(h) * rows_pad + i] = make_float2(i < T ? -lse[int64_t(h) * T + i] * inv_scale : 0.f, -acc);
            }
        }
    }
}

// Split x into three bf16 parts whose sum is x to about 2^-24 relative: the packed (hi, mid) and (lo, 0) words.
__device__ __forceinline__ uint2 split3_bf16(float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
    return make_uint2(uint32_t(__bfloat16_as_ushort(h)) | (uint32_t(__bfloat16_as_ushort(m)) << 16),
                      uint32_t(__bfloat16_as_ushort(l)));
}

// ------------------------------------------------------------------------------------------------- main kernel
struct BwdSmem {
    static constexpr int TILE = 128 * BWD_D * 2;         // 128 rows x d, bf16 (K, V, Q, dO)
    static constexpr int CHUNK = 128 * 64 * 2;           // one 64-column 128-byte-swizzled chunk of such a tile
    static constexpr int QSTAGES = 2;
    static constexpr int AUG = 128 * 16 * 2;             // 128 rows x 16 bf16, no-swizzle core-matrix layout
    static constexpr int AUG_LBO = 128, AUG_SBO = 256;   // next 8 columns / next 8 rows
    alignas(1024) uint8_t k[TILE];
    alignas(1024) uint8_t v[TILE];
    alignas(1024) uint8_t q[QSTAGES][TILE];
    alignas(1024) uint8_t dout[QSTAGES][TILE];
    alignas(1024) uint8_t aug_ones[AUG];                 // key side of the extra slice: (1, 1, 1, 0, ...)
    alignas(1024) uint8_t aug_q[QSTAGES][AUG];           // query side for S^T: split(-lse / scale)
    alignas(1024) uint8_t aug_do[QSTAGES][AUG];          // query side for dP^T: split(-D)
    uint64_t k_full, k_empty, v_full, v_empty, dkv_full, dkv_free;
    uint64_t q_full[QSTAGES], q_empty[QSTAGES], do_full[QSTAGES], do_empty[QSTAGES];
    uint64_t s_full, s_free, dp_full, dp_free, p_ready, ds_ready;
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(BwdSmem) + 1024 <= 232448, "dK/dV kernel shared memory exceeds 227 KB");

struct BwdItem {
    KTile t;
    int qa, qb, split, kh;
    int slot0;        // dS slot of the chunk's first step
};

// Work item -> (work chunk, kv head). Items run in groups of up to four kv heads; within a group, chunks in cost
// order with the group's heads interleaved. Cost order keeps the static round-robin balanced; the head groups keep
// the Q/dO tiles that concurrently running items read (those of the group's q heads) small enough to stay in L2.
__device__ __forceinline__ int2 bwd_item_split(int item, int n_bw, int hkv) {
    const int G = (hkv % 4 == 0) ? 4 : (hkv % 2 == 0 ? 2 : 1);
    const int per = n_bw * G;
    const int grp = item / per, pos = item % per;
    return make_int2(pos / G, grp * G + pos % G);
}

__device__ __forceinline__ BwdItem bwd_decode(const void *meta, const MetaHeader &hd, int item, int hkv) {
    const int2 bk = bwd_item_split(item, hd.n_bw, hkv);
    const BWork w = meta_ptr<BWork>(meta, hd.off_bw)[bk.x];
    BwdItem it;
    it.kh = bk.y;
    it.t = KTile{};
    it.t.row0 = w.row0;
    it.t.gstart = w.gstart;
    it.t.glen = w.glen;
    it.qa = w.qa;
    it.qb = w.qb;
    it.split = w.split;
    it.slot0 = w.slot0;
    return it;
}

// Byte offset of row r, column 0 in a 128 x 16 bf16 no-swizzle K-major tile (8-row x 16-byte core matrices).
__device__ __forceinline__ uint32_t aug_row_off(int r) { return (r >> 3) * 256 + (r & 7) * 16; }

__device__ __forceinline__ void red_add_v4(float *addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// 64 columns of dK (dS^T carried the scale) or dV of one key row, from registers: bf16 for an unsplit key tile,
// fp32 adds into the workspace for a split one.
__device__ __forceinline__ void bwd_store_kv64(const uint32_t (&a)[32], const uint32_t (&b)[32], bool split,
                                               float *acc, __nv_bfloat16 *dst, bool v8) {
    if (split) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            red_add_v4(acc + 4 * e, __uint_as_float(a[4 * e]), __uint_as_float(a[4 * e + 1]),
                       __uint_as_float(a[4 * e + 2]), __uint_as_float(a[4 * e + 3]));
#pragma unroll
        for (int e = 0; e < 8; ++e)
            red_add_v4(acc + 32 + 4 * e, __uint_as_float(b[4 * e]), __uint_as_float(b[4 * e + 1]),
                       __uint_as_float(b[4 * e + 2]), __uint_as_float(b[4 * e + 3]));
    } else {                                                   // 128 bytes: four 32-byte stores
        auto pk = [](const uint32_t *x, int i) { return pack_bf16x2(__uint_as_float(x[i]), __uint_as_float(x[i + 1])); };
#pragma unroll
        for (int e = 0; e < 2; ++e)
            st_global_32(dst + 16 * e, v8, pk(a, 16 * e), pk(a, 16 * e + 2), pk(a, 16 * e + 4), pk(a, 16 * e + 6),
                         pk(a, 16 * e + 8), pk(a, 16 * e + 10), pk(a, 16 * e + 12), pk(a, 16 * e + 14));
#pragma unroll
        for (int e = 0; e < 2; ++e)
            st_global_32(dst + 32 + 16 * e, v8, pk(b, 16 * e), pk(b, 16 * e + 2), pk(b, 16 * e + 4), pk(b, 16 * e + 6),
                         pk(b, 16 * e + 8), pk(b, 16 * e + 10), pk(b, 16 * e + 12), pk(b, 16 * e + 14));
    }
}

__global__ void __launch_bounds__(BWD_THREADS, 1)
k_bwd_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
         const void *__restrict__ meta, const float2 *__restrict__ ldg,
         float *__restrict__ dk_acc, float *__restrict__ dv_acc,
         __nv_bfloat16 *__restrict__ dK, __nv_bfloat16 *__restrict__ dV, int hq, int hkv, int64_t rows_pad,
         float scale, float sl2, __nv_bfloat16 *__restrict__ ds_buf, int64_t ds_cap) {
    extern __shared__ uint8_t smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
    const int r = hq / hkv;
    const int n_items = hd.n_bw * hkv;
    volatile int *abort_flag = &sm.abort_flag;

    if (threadIdx.x == 0) {
        mbar_init(&sm.k_full, 1);
        mbar_init(&sm.k_empty, 1);
        mbar_init(&sm.v_full, 1);
        mbar_init(&sm.v_empty, 1);
        mbar_init(&sm.dkv_full, 1);
        mbar_init(&sm.dkv_free, 256);
        for (int b = 0; b < BwdSmem::QSTAGES; ++b) {
            mbar_init(&sm.q_full[b], 32);
            mbar_init(&sm.q_empty[b], 1);
            mbar_init(&sm.do_full[b], 32);
            mbar_init(&sm.do_empty[b], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, 256);                      // the gradient warps have read S^T(g)
        mbar_init(&sm.dp_full, 1);
        mbar_init(&sm.dp_free, 1);                       // dV(g) and dK(g) have read P^T(g), dS^T(g) (dP columns)
        mbar_init(&sm.p_ready, 256);
        mbar_init(&sm.ds_ready, 256);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    {   // extra-slice tiles: zeros everywhere, ones in columns 0-2 of the key-side tile
        uint4 *z = reinterpret_cast<uint4 *>(sm.aug_ones);
        for (int i = threadIdx.x; i < (1 + 2 * BwdSmem::QSTAGES) * BwdSmem::AUG / 16; i += blockDim.x)
            z[i] = make_uint4(0, 0, 0, 0);
        __syncthreads();
        if (threadIdx.x < 128) {
            const uint32_t one = 0x3f80u;                          // bf16 1.0
            *reinterpret_cast<uint2 *>(sm.aug_ones + aug_row_off(threadIdx.x)) =
                make_uint2(one | (one << 16), one);
        }
        fence_proxy_async_smem();
    }
    if (warp == 9) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdO);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 384;

    if (hd.dev_err != 0) {
        // nothing to do: the metadata builder rejected its input
    } else if (warp == 8) {
        // ------------------------------------------------------------------ producer warp
        // Loads in the order the MMAs need them: K of the item, then per step Q (with its extra-slice tile), V (on
        // the item's first step) and dO (with its extra-slice tile). Q and dO have separate stages, so each is
        // reloaded as soon as its own last MMA (dK, dV) has read it.
        uint32_t g = 0, it_n = 0;
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it_n) {
            const BwdItem w = bwd_decode(meta, hd, item, hkv);
            const int n = (w.qb - w.qa) * r;
            auto step_h = [&](int t) { return w.kh * r + t % r; };
            auto step_x0 = [&](int t) { return w.t.gstart + (w.qa + t / r) * BWD_BM; };
            if (lane == 0) {
                const int nxt = item + int(gridDim.x);
                if (nxt < n_items) {                                   // the next item's K/V into L2
                    const BwdItem wn = bwd_decode(meta, hd, nxt, hkv);
                    for (int c = 0; c < BWD_D / 64; ++c) {
                        tma_prefetch_3d(&tmK, c * 64, wn.kh, wn.t.row0);
                        tma_prefetch_3d(&tmV, c * 64, wn.kh, wn.t.row0);
                    }
                }
                if (!bwait(&sm.k_empty, (it_n & 1) ^ 1, abort_flag)) goto done;
                mbar_arrive_expect_tx(&sm.k_full, BwdSmem::TILE);
                for (int c = 0; c < BWD_D / 64; ++c)
                    tma_load_3d(sm.k + c * BwdSmem::CHUNK, &tmK, c * 64, w.kh, w.t.row0, &sm.k_full);
                for (int t = 0; t < 2 && t < n; ++t)
                    for (int c = 0; c < BWD_D / 64; ++c) {
                        tma_prefetch_3d(&tmQ, c * 64, step_h(t), step_x0(t));
                        tma_prefetch_3d(&tmdO, c * 64, step_h(t), step_x0(t));
                    }
            }
            float2 lv[4];                                              // rows lane + 32u of the current step
#pragma unroll
            for (int u = 0; u < 4; ++u) lv[u] = ldg[int64_t(step_h(0)) * rows_pad + step_x0(0) + lane + 32 * u];
            for (int t = 0; t < n; ++t, ++g) {
                const int st = g % BwdSmem::QSTAGES;
                const uint32_t ph = ((g / BwdSmem::QSTAGES) & 1) ^ 1;
                const int h = step_h(t);
                const int x0 = step_x0(t);
                // next step's values and (two steps ahead) its tiles: their latency hides behind this step
                float2 nv[4];
                if (t + 1 < n) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) nv[u] = ldg[int64_t(step_h(t + 1)) * rows_pad + step_x0(t + 1) + lane + 32 * u];
                }
                if (lane == 0 && t + 2 < n)
                    for (int c = 0; c < BWD_D / 64; ++c) {
                        tma_prefetch_3d(&tmQ, c * 64, step_h(t + 2), step_x0(t + 2));
                        tma_prefetch_3d(&tmdO, c * 64, step_h(t + 2), step_x0(t + 2));
                    }
                // Q(t) and its slice split(-lse / scale)
                if (!bwait(&sm.q_empty[st], ph, abort_flag)) goto done;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint2 *>(sm.aug_q[st] + aug_row_off(lane + 32 * u)) = split3_bf16(lv[u].x);
                fence_proxy_async_smem();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm.q_full[st], BwdSmem::TILE);
                    for (int c = 0; c < BWD_D / 64; ++c)
                        tma_load_3d(sm.q[st] + c * BwdSmem::CHUNK, &tmQ, c * 64, h, x0, &sm.q_full[st]);
                } else {
                    mbar_arrive(&sm.q_full[st]);
                }
                if (t == 0 && lane == 0) {                             // V of the item (feeds dP^T only)
                    if (!bwait(&sm.v_empty, (it_n & 1) ^ 1, abort_flag)) goto done;
                    mbar_arrive_expect_tx(&sm.v_full, BwdSmem::TILE);
                    for (int c = 0; c < BWD_D / 64; ++c)
                        tma_load_3d(sm.v + c * BwdSmem::CHUNK, &tmV, c * 64, w.kh, w.t.row0, &sm.v_full);
                }
                // dO(t) and its slice split(-D)
                if (!bwait(&sm.do_empty[st], ph, abort_flag)) goto done;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    *reinterpret_cast<uint2 *>(sm.aug_do[st] + aug_row_off(lane + 32 * u)) = split3_bf16(lv[u].y);
                fence_proxy_async_smem();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm.do_full[st], BwdSmem::TILE);
                    for (int c = 0; c < BWD_D / 64; ++c)
                        tma_load_3d(sm.dout[st] + c * BwdSmem::CHUNK, &tmdO, c * 64, h, x0, &sm.do_full[st]);
                } else {
                    mbar_arrive(&sm.do_full[st]);
                }
                if (t + 1 < n) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) lv[u] = nv[u];
                }
            }
        }
    } else if (warp == 9 || warp == 10) {
        // ------------------------------------------------------------------ MMA issuers (one thread each)
        // Issuing one MMA takes a thread about 50 cycles, close to the 64 an N = 128 MMA runs, so a single issuer
        // that also polls barriers leaves the tensor pipe idle; two issuers overlap one's polls with the other's
        // MMAs. Warp 9 issues the score products, warp 10 the gradient products:
        //   warp 9:  S^T(g+1) once the gradient warps hold S^T(g) in registers (s_free), then dP^T(g+1) once dV(g)
        //            and dK(g) have read P^T(g) and dS^T(g) from the dP columns (dp_free);
        //   warp 10: dV(g) once P^T(g) is in TMEM (p_ready), then dK(g) once dS^T(g) is (ds_ready).
        constexpr uint32_t ID_SDP = idesc_bf16(128, BWD_BM, 0, 0);     // S^T, dP^T (both K-major)
        constexpr uint32_t ID_KV = idesc_bf16(128, BWD_D, 0, 1);       // dK, dV (A TMEM, B MN-major)
        constexpr uint32_t TB = BwdSmem::TILE, AB = BwdSmem::AUG;
        const BWork *bws = meta_ptr<BWork>(meta, hd.off_bw);
        auto item_steps = [&](int it) { const BWork b = bws[bwd_item_split(it, hd.n_bw, hkv).x]; return (b.qb - b.qa) * r; };
        if (warp == 9 && lane == 0 && int(blockIdx.x) < n_items) {
            // descriptors built once; a stage is a constant stride away (desc_adv)
            const uint64_t k_desc = smem_desc(smem_u32(sm.k), 16, 1024);
            const uint64_t v_desc = smem_desc(smem_u32(sm.v), 16, 1024);
            const uint64_t q_desc = smem_desc(smem_u32(sm.q[0]), 16, 1024);
            const uint64_t do_desc = smem_desc(smem_u32(sm.dout[0]), 16, 1024);
            const uint64_t ones_desc = smem_desc(smem_u32(sm.aug_ones), BwdSmem::AUG_LBO, BwdSmem::AUG_SBO, 0);
            const uint64_t augq_desc = smem_desc(smem_u32(sm.aug_q[0]), BwdSmem::AUG_LBO, BwdSmem::AUG_SBO, 0);
            const uint64_t augdo_desc = smem_desc(smem_u32(sm.aug_do[0]), BwdSmem::AUG_LBO, BwdSmem::AUG_SBO, 0);
            auto issue_kk = [&](uint32_t col, uint64_t a, uint64_t b, uint64_t aug) {
                const uint32_t d = tmem + col;
#pragma unroll
                for (int kk = 0; kk < BWD_D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * BwdSmem::CHUNK + (kk & 3) * 32;
                    umma_ss(d, desc_adv(a, off), desc_adv(b, off), ID_SDP, kk > 0);
                }
                // the extra slice: + (1,1,1) . split(value of the query row)
                umma_ss(d, ones_desc, aug, ID_SDP, 1u);
            };
            // S^T(gg) (first of its item: after K lands) and dP^T(gg)
            auto issue_s = [&](uint32_t gg, bool first, uint32_t item_par, bool last) -> bool {
                const int st = gg % BwdSmem::QSTAGES;
                if (first && !bwait(&sm.k_full, item_par, abort_flag)) return false;
                if (!bwait(&sm.q_full[st], (gg / BwdSmem::QSTAGES) & 1, abort_flag)) return false;
                tc_fence_after();
                issue_kk(COL_S, k_desc, q_desc + uint64_t(st) * (TB >> 4), augq_desc + uint64_t(st) * (AB >> 4));
                umma_commit(&sm.s_full);
                if (last) umma_commit(&sm.k_empty);                  // K feeds S^T only
                return true;
            };
            auto issue_dp = [&](uint32_t gg, bool first, uint32_t item_par, bool last) -> bool {
                const int st = gg % BwdSmem::QSTAGES;
                if (first && !bwait(&sm.v_full, item_par, abort_flag)) return false;
                if (!bwait(&sm.do_full[st], (gg / BwdSmem::QSTAGES) & 1, abort_flag)) return false;
                tc_fence_after();
                issue_kk(COL_DP, v_desc, do_desc + uint64_t(st) * (TB >> 4), augdo_desc + uint64_t(st) * (AB >> 4));
                umma_commit(&sm.dp_full);
                if (last) umma_commit(&sm.v_empty);                  // V feeds dP^T only
                return true;
            };
            int item = blockIdx.x, n = item_steps(item), t = 0;
            uint32_t g = 0, it_n = 0;
            if (!issue_s(0, true, 0, n == 1)) goto done;
            if (!issue_dp(0, true, 0, n == 1)) goto done;
            for (;;) {
                int item2 = item, t2 = t + 1, n2 = n;
                if (t2 == n) {
                    item2 = item + int(gridDim.x);
                    t2 = 0;
                    n2 = item2 < n_items ? item_steps(item2) : 0;
                }
                if (item2 >= n_items) break;
                const bool next_first = t2 == 0;
                const uint32_t par2 = (it_n + (next_first ? 1u : 0u)) & 1;
                if (!bwait(&sm.s_free, g & 1, abort_flag)) goto done;      // S^T(g) is in registers
                if (!issue_s(g + 1, next_first, par2, t2 + 1 == n2)) goto done;
                if (!bwait(&sm.dp_free, g & 1, abort_flag)) goto done;     // dV(g), dK(g) read the dP columns
                if (!issue_dp(g + 1, next_first, par2, t2 + 1 == n2)) goto done;
                ++g;
                if (next_first) ++it_n;
                item = item2;
                t = t2;
                n = n2;
            }
        } else if (warp == 10 && lane == 0) {
            const uint64_t qn_desc = smem_desc(smem_u32(sm.q[0]), BwdSmem::CHUNK, 1024);      // N-major (dK)
            const uint64_t don_desc = smem_desc(smem_u32(sm.dout[0]), BwdSmem::CHUNK, 1024);  // N-major (dV)
            uint32_t g = 0, it_n = 0;
            for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it_n) {
                const int n = item_steps(item);
                for (int t = 0; t < n; ++t, ++g) {
                    const int st = g % BwdSmem::QSTAGES;
                    const uint64_t bq = qn_desc + uint64_t(st) * (TB >> 4), bdo = don_desc + uint64_t(st) * (TB >> 4);
                    const uint32_t acc0 = t > 0 ? 1u : 0u;
                    // dV += P^T dO as soon as P^T is in the dP columns (the epilogue has read the last item's dV)
                    if (!bwait(&sm.p_ready, g & 1, abort_flag)) goto done;
                    if (t == 0 && !bwait(&sm.dkv_free, (it_n & 1) ^ 1, abort_flag)) goto done;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BWD_BM / 16; ++kk)
                        umma_ts(tmem + COL_DV, tmem + COL_DP + 64 * (kk >> 2) + 8 * (kk & 3),
                                desc_adv(bdo, kk * 2048), ID_KV, kk > 0 ? 1u : acc0);
                    umma_commit(&sm.do_empty[st]);
                    // dK += dS^T Q once dS^T is in the dP columns
                    if (!bwait(&sm.ds_ready, g & 1, abort_flag)) goto done;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < BWD_BM / 16; ++kk)
                        umma_ts(tmem + COL_DK, tmem + COL_DP + 64 * (kk >> 2) + 32 + 8 * (kk & 3),
                                desc_adv(bq, kk * 2048), ID_KV, kk > 0 ? 1u : acc0);
                    umma_commit(&sm.q_empty[st]);
                    umma_commit(&sm.dp_free);
                    if (t + 1 == n) umma_commit(&sm.dkv_full);
                }
            }
        }
    } else {
        // ------------------------------------------------------------------ gradient warpgroups (warps 0-7)
        // Warpgroup x handles query columns [64x, 64x+64) of every step (TMEM lane = key row). Per step: read S^T
        // (the next step's S^T may then be issued), P^T = exp2(S'^T scale log2 e); read dP^T; P^T (bf16) into the
        // first 32 of the 64 dP columns it reads -> p_ready (dV may start); dS^T = scale P^T dP'^T (bf16) into the
        // last 32 -> ds_ready (dK may start). The next step's dP^T waits for both.
        const int wx = warp >> 2;                                      // column half
        const int wl = warp & 3;
        const int jr = wl * 32 + lane;                                 // TMEM lane: key row
        const uint32_t lane_off = uint32_t(wl * 32) << 16;
        const int cb = 64 * wx;                                        // first query column of this half
        // dS kept for the dQ kernel: slot s holds the step's dS^T tile, [128 key rows][128 query columns] bf16
        const bool keep_ds = ds_buf != nullptr && int64_t(hd.n_slots) * hkv <= ds_cap;
        const bool out_v8 = aligned32(wx == 0 ? dK : dV);              // rows are 256 bytes: the base decides
        uint32_t g = 0, it_n = 0;
        const int32_t *key_end = meta_ptr<int32_t>(meta, hd.off_key_end);
        // Item epilogue, run inside the next item's first step (after its P, before its dS), when dK/dV of the
        // item have long been complete: warpgroup 0 takes dK, warpgroup 1 dV, 64 columns at a time; the
        // accumulator is released as soon as the last columns are in registers.
        bool ep_yin = false, ep_split = false;
        int64_t ep_row = 0;
        auto epilogue = [&](uint32_t en) -> bool {
            if (!bwait(&sm.dkv_full, en & 1, abort_flag)) return false;
            tc_fence_after();
            const uint32_t src = tmem + lane_off + (wx == 0 ? COL_DK : COL_DV);
            float *acc = (wx == 0 ? dk_acc : dv_acc) + ep_row;
            __nv_bfloat16 *dst = (wx == 0 ? dK : dV) + ep_row;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t a[32], b[32];
                tmem_ld32(src + 64 * half, a);
                tmem_ld32(src + 64 * half + 32, b);
                tmem_wait_ld(a, b);
                if (half == 1) {                                       // the accumulator is no longer needed
                    tc_fence_before();
                    mbar_arrive(&sm.dkv_free);
                }
                if (ep_yin) bwd_store_kv64(a, b, ep_split, acc + 64 * half, dst + 64 * half, out_v8);
            }
            return true;
        };
        auto key_end_of = [&](const BwdItem &b) {
            const int yy = b.t.row0 + jr;
            return yy < b.t.gstart + b.t.glen ? key_end[yy] : yy;
        };
        BwdItem wn{};
        int ken = 0;
        if (blockIdx.x < n_items) {
            wn = bwd_decode(meta, hd, blockIdx.x, hkv);
            ken = key_end_of(wn);
        }
        for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it_n) {
            const BwdItem w = wn;
            const int ke = ken;                                        // queries [y, ke) attend key y
            const int nxt = item + gridDim.x;
            if (nxt < n_items) wn = bwd_decode(meta, hd, nxt, hkv);
            const int n = (w.qb - w.qa) * r;
            const int y = w.t.row0 + jr;
            const int gend = w.t.gstart + w.t.glen;
            const bool yin = y < gend;
            for (int t = 0; t < n; ++t, ++g) {
                const int x0 = w.t.gstart + (w.qa + t / r) * BWD_BM;
                const int lo = y - x0 - cb, hi = ke - x0 - cb;         // allowed columns [lo, hi) of this half
                const bool all_in = __all_sync(0xffffffffu, lo <= 0 && hi >= 64);
                // P^T = exp2(S'^T * scale * log2 e) (S' already holds s - lse / scale), packed bf16
                uint32_t pk[32];
                if (!bwait(&sm.s_full, g & 1, abort_flag)) goto done;
                tc_fence_after();
                {
                    uint32_t a0[32], a1[32];
                    tmem_ld32(tmem + lane_off + COL_S + cb, a0);
                    tmem_ld32(tmem + lane_off + COL_S + cb + 32, a1);
                    tmem_wait_ld(a0, a1);
                    tc_fence_before();
                    mbar_arrive(&sm.s_free);                           // the next step's S^T may overwrite it
                    if (all_in) {
                        const float2 sl2v = make_float2(sl2, sl2);
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const uint32_t u0 = e < 16 ? a0[2 * e] : a1[2 * e - 32];
                            const uint32_t u1 = e < 16 ? a0[2 * e + 1] : a1[2 * e - 31];
                            const float2 x = fmul2(make_float2(__uint_as_float(u0), __uint_as_float(u1)), sl2v);
                            pk[e] = pack_bf16x2(ex2_approx(x.x), ex2_approx(x.y));
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int c = 2 * e;
                            const uint32_t u0 = e < 16 ? a0[2 * e] : a1[2 * e - 32];
                            const uint32_t u1 = e < 16 ? a0[2 * e + 1] : a1[2 * e - 31];
                            const float p0 = (c >= lo && c < hi) ? ex2_approx(__uint_as_float(u0) * sl2) : 0.f;
                            const float p1 = (c + 1 >= lo && c + 1 < hi) ? ex2_approx(__uint_as_float(u1) * sl2) : 0.f;
                            pk[e] = pack_bf16x2(p0, p1);
                        }
                    }
                }
                if (t == 0) {
                    if (it_n > 0 && !epilogue(it_n - 1)) goto done;
                    ep_yin = yin;
                    ep_split = w.split;
                    ep_row = (int64_t(y) * hkv + w.kh) * BWD_D;
                    if (nxt < n_items) ken = key_end_of(wn);
                }
                // dP^T, then P^T (bf16) into the first 32 of the 64 dP columns this warpgroup reads (dV may start),
                // then dS^T = scale P^T dP'^T (dP' = dP - D already) into the last 32 (dK may start)
                if (!bwait(&sm.dp_full, g & 1, abort_flag)) goto done;
                tc_fence_after();
                {
                    uint32_t ds[32];
                    const float2 sc = make_float2(scale, scale);
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t a0[32];
                        tmem_ld32(tmem + lane_off + COL_DP + cb + 32 * hf, a0);
                        tmem_wait_ld(a0);
                        if (hf == 0) {                                 // these columns are read: P^T goes there
                            tmem_st32(tmem + lane_off + COL_DP + cb, pk);
                            tmem_wait_st();
                            tc_fence_before();
                            mbar_arrive(&sm.p_ready);
                        }
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const uint32_t p = pk[16 * hf + e];
                            const float2 d2 = fmul2(fmul2(make_float2(bf16lo(p), bf16hi(p)), sc),
                                                    make_float2(__uint_as_float(a0[2 * e]), __uint_as_float(a0[2 * e + 1])));
                            ds[16 * hf + e] = pack_bf16x2(d2.x, d2.y);
                        }
                    }
                    tmem_st32(tmem + lane_off + COL_DP + cb + 32, ds);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&sm.ds_ready);
                    if (keep_ds) {   // this key row's 64 query columns of dS, after dK(g) has been released
                        const int64_t slot = int64_t(w.kh) * hd.n_slots + w.slot0 + t;   // slots: kv head major
                        __nv_bfloat16 *dst = ds_buf + (slot * BWD_BN + jr) * BWD_BM + cb;   // 32-byte aligned
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            st_global_32(dst + 16 * e, true, ds[8 * e], ds[8 * e + 1], ds[8 * e + 2], ds[8 * e + 3],
                                         ds[8 * e + 4], ds[8 * e + 5], ds[8 * e + 6], ds[8 * e + 7]);
                    }
                }
            }
        }
        if (it_n > 0 && !epilogue(it_n - 1)) goto done;
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------------- convert
// dK/dV rows of split key tiles = bf16(fp32 accumulators). A unit is 16 rows of one key tile (contiguous rows).
__global__ void k_bwd_convert(const void *__restrict__ meta, const float *__restrict__ dk_acc,
                              const float *__restrict__ dv_acc, __nv_bfloat16 *__restrict__ dK,
                              __nv_bfloat16 *__restrict__ dV, int hkv) {
    const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
    if (hd.dev_err || hd.n_split == 0) return;
    const KTile *kts = meta_ptr<KTile>(meta, hd.off_kt);
    const int per_row = hkv * (BWD_D / 4);                             // float4 (four elements) per row
    for (int u = blockIdx.x; u < hd.n_kt * 8; u += gridDim.x) {
        const KTile t = kts[u >> 3];
        if (t.nch <= 1) continue;
        const int r0 = (u & 7) * 16;
        const int rows = min(16, t.gstart + t.glen - t.row0 - r0);
        if (rows <= 0) continue;
        const int64_t base = (int64_t(t.row0) + r0) * per_row;
        for (int which = 0; which < 2; ++which) {
            const float4 *src = reinterpret_cast<const float4 *>(which ? dv_acc : dk_acc) + base;
            uint2 *dst = reinterpret_cast<uint2 *>(which ? dV : dK) + base;
            for (int e = threadIdx.x; e < rows * per_row; e += blockDim.x) {
                const float4 a = src[e];
                __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
                uint2 v;
                v.x = *reinterpret_cast<uint32_t *>(&lo);
                v.y = *reinterpret_cast<uint32_t *>(&hi);
                dst[e] = v;
            }
        }
    }
}

// ------------------------------------------------------------------------------------------------- launcher
typedef pp_status (*MakeMapFn)(CUtensorMap *, const void *, int64_t, int, int, int);
typedef pp_status (*FailFn)(pp_status, const char *, ...);

// Bytes of one kept dS tile (one backward step) and the alignment of the dS region after the base workspace.
constexpr int64_t BWD_DS_TILE_BYTES = int64_t(BWD_BN) * BWD_BM * 2;
constexpr int64_t BWD_DS_ALIGN = 1024;

typedef pp_status (*MakeMapBoxFn)(CUtensorMap *, const void *, int64_t, int, int, int, int);

// ws_bytes beyond the base layout holds kept dS tiles: if all the batch's steps fit, the key-side kernel writes them
// and k_bwd_dq_ds forms dQ from them; otherwise k_bwd_dq recomputes S and dP. Both dQ kernels are launched and the
// one whose case does not hold returns at once (the slot count is only known on the device).
inline pp_status launch_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                            const void *dout, const void *meta, int64_t T, int hq, int hkv, int d, float scale,
                            void *dq, void *dk, void *dv, void *workspace, int64_t ws_bytes, int sm_count,
                            cudaStream_t s, MakeMapFn make_map, MakeMapBoxFn make_map_box, FailFn fail) {
    if (d != BWD_D) return fail(PP_ERR_UNSUPPORTED, "backward supports head dim 128 only (got %d)", d);
    const BwdWorkspace L = bwd_workspace_layout(T, hq, hkv, d);
    char *ws = static_cast<char *>(workspace);
    float2 *ldg = reinterpret_cast<float2 *>(ws + L.off_delta);
    float *dk_acc = reinterpret_cast<float *>(ws + L.off_dk);
    float *dv_acc = reinterpret_cast<float *>(ws + L.off_dv);
    const void *ptrs[8] = {q, k, v, o, dout, dq, dk, dv};
    for (const void *p : ptrs)
        if (reinterpret_cast<uintptr_t>(p) % 16) return fail(PP_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    CUtensorMap mq, mk, mv, mdo, mds;
    pp_status st;
    if ((st = make_map(&mq, q, T, hq, d, BWD_BM)) != PP_OK) return st;
    if ((st = make_map(&mk, k, T, hkv, d, BWD_BN)) != PP_OK) return st;
    if ((st = make_map(&mv, v, T, hkv, d, BWD_BN)) != PP_OK) return st;
    if ((st = make_map(&mdo, dout, T, hq, d, BWD_BM)) != PP_OK) return st;
    // the dS region: what the workspace holds past the base layout, in whole tiles
    const int64_t ds_off = (L.total + BWD_DS_ALIGN - 1) / BWD_DS_ALIGN * BWD_DS_ALIGN;
    int64_t ds_cap = ws_bytes > ds_off ? (ws_bytes - ds_off) / BWD_DS_TILE_BYTES : 0;
    if (ds_cap > (int64_t(1) << 24)) ds_cap = int64_t(1) << 24;       // TMA row coordinate stays below 2^31
    // the schedule builder counts steps and slot offsets in int32: keep no dS tiles where a batch of T tokens could
    // have more (T above about 4.2 M tokens at r = 4)
    if (bwd_steps_bound(T, hq / hkv) > int64_t(0x7fffffff)) ds_cap = 0;
    __nv_bfloat16 *ds_buf = ds_cap > 0 ? reinterpret_cast<__nv_bfloat16 *>(ws + ds_off) : nullptr;
    if (ds_buf && (st = make_map_box(&mds, ds_buf, ds_cap * BWD_BN, 1, BWD_BM, 1, BWD_BN)) != PP_OK) return st;
    cudaError_t e;
    k_bwd_pre<<<sm_count * 8, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(o),
                                           static_cast<const __nv_bfloat16 *>(dout), lse, ldg, T, L.rows_pad, hq,
                                           1.f / scale, meta, dk_acc, dv_acc, hkv);
    if ((e = cudaGetLastError()) != cudaSuccess) return fail(PP_ERR_CUDA, "k_bwd_pre: %s", cudaGetErrorString(e));
    const size_t smem = sizeof(BwdSmem) + 1024;
    if ((e = cudaFuncSetAttribute(k_bwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem))) != cudaSuccess)
        return fail(PP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    k_bwd_tc<<<sm_count, BWD_THREADS, smem, s>>>(mq, mk, mv, mdo, meta, ldg, dk_acc, dv_acc,
                                                 static_cast<__nv_bfloat16 *>(dk), static_cast<__nv_bfloat16 *>(dv),
                                                 hq, hkv, L.rows_pad, scale, scale * 1.4426950408889634f, ds_buf,
                                                 ds_cap);
    if ((e = cudaGetLastError()) != cudaSuccess) return fail(PP_ERR_CUDA, "k_bwd_tc: %s", cudaGetErrorString(e));
    const size_t smem_dq = sizeof(DqSmem) + 1024;
    if ((e = cudaFuncSetAttribute(k_bwd_dq, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_dq))) != cudaSuccess)
        return fail(PP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    k_bwd_dq<<<sm_count, DQ_THREADS, smem_dq, s>>>(mq, mk, mv, mdo, meta, ldg, static_cast<__nv_bfloat16 *>(dq),
                                                   hq, hkv, L.rows_pad, scale, scale * 1.4426950408889634f, ds_buf,
                                                   ds_cap);
    if ((e = cudaGetLastError()) != cudaSuccess) return fail(PP_ERR_CUDA, "k_bwd_dq: %s", cudaGetErrorString(e));
    if (ds_buf) {
        const size_t smem_ds = sizeof(DqsSmem) + 1024;
        if ((e = cudaFuncSetAttribute(k_bwd_dq_ds, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_ds))) !=
            cudaSuccess)
            return fail(PP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        k_bwd_dq_ds<<<sm_count, DQS_THREADS, smem_ds, s>>>(mds, mk, meta, static_cast<__nv_bfloat16 *>(dq), hq, hkv,
                                                            ds_buf, ds_cap);
        if ((e = cudaGetLastError()) != cudaSuccess) return fail(PP_ERR_CUDA, "k_bwd_dq_ds: %s", cudaGetErrorString(e));
    }
    k_bwd_convert<<<sm_count * 8, 256, 0, s>>>(meta, dk_acc, dv_acc, static_cast<__nv_bfloat16 *>(dk),
                                               static_cast<__nv_bfloat16 *>(dv), hkv);
    if ((e = cudaGetLastError()) != cudaSuccess) return fail(PP_ERR_CUDA, "k_bwd_convert: %s", cudaGetErrorString(e));
    return PP_OK;
}

}  // namespace pp
