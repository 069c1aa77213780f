// pp_decode.cuh - decode-time attention over a group-contiguous KV cache (pp.h, pp_decode_attn).
//
// The cache holds, group by group, the prefix's K/V rows and then each response's rows, the newest token of each
// response last ("PackInfer" abstract: group-contiguous KV, so a shared prefix is read once; "Preference Packing":
// responses share the prompt's attention). Each response has one query, its newest token, which attends to the
// group's prefix and to its own rows, under the same mask as the packed prefill.
// Flash-decoding over 128-key chunks of every cache segment:
//   k_dec_plan   one block: segment -> group, chunk counts, (chunk, query) record offsets and job offsets (scans).
//   k_dec_chunk  persistent tcgen05 kernel over jobs (chunk, kv head, query block). A job's query block is every
//                query that sees the chunk (all responses of the group for a prefix chunk, one response for a
//                response chunk) times the r q heads of the kv head, up to 128 rows, gathered by one 3-D TMA box
//                from q [n_resp, hq, d]. S = Q K^T and O = P V run on the tensor cores (M = 128 query rows, N = 128
//                keys, then N = d); two softmax warpgroups take alternate jobs, each thread one query row. A prefix
//                chunk is therefore read from
//                HBM once per group (per query block), not once per response. Each job writes an fp32 record
//                (max, sum, un-normalised O) per valid query row.
//   k_dec_combine one warp per (response, q head): merges its records (the group's prefix chunks, its own chunks).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "pp_build.cuh"     // block_exclusive_scan, upper_bound_i32, g_dev_err
#include "pp_ptx.cuh"
#include "pp_attn_fwd.cuh"  // bwait

namespace pp {

constexpr int DEC_CH = 128;           // keys per chunk (the MMA N of S, the K of P V)
constexpr int DEC_D = 128;            // head dim
constexpr int DEC_REC = 136;          // floats per record: max (base 2), sum, six pad, O[128] (32-byte aligned)
constexpr int DEC_REC_O = 8;          // offset of O in a record
constexpr int DEC_STAGES = 3;         // K and V chunk rings
constexpr int DEC_THREADS = 320;      // warps 0-7 softmax / records (two warpgroups), warp 8 TMA, warp 9 MMA

// Plan layout in the workspace (int32 sections, sizes from G and nseg).
struct DecPlan {
    int64_t off_first_seg;   // [G + 1] first segment of each group (exclusive scan of 1 + k_g)
    int64_t off_seg_group;   // [nseg]
    int64_t off_unit_off;    // [nseg + 1] chunks before each segment
    int64_t off_pair_off;    // [nseg + 1] (chunk, query) records before each segment
    int64_t off_job_off;     // [nseg + 1] jobs (chunk, query block) before each segment
    int64_t off_counts;      // [4]: units, records, ok (1 if the plan fits), jobs
    int64_t off_jobs;        // DecJobRec[max_pairs]: every job decoded once (jobs <= records)
    int64_t off_resp;        // DecRespRec[nseg - G]: where each response's records lie
    int64_t off_part;        // fp32 records: [pairs][hq][DEC_REC]
    int64_t total;
    int64_t max_pairs;       // records the workspace holds
};

__host__ __device__ inline int64_t dec_a256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Section offsets for a workspace that holds max_pairs (chunk, query) records. The exact number of records is the
// sum over prefixes of nch * k_g plus the sum over responses of nch, nch = ceil(len / DEC_CH); the host sizing call
// computes it from host copies of the descriptors.
__host__ inline DecPlan dec_plan_layout(int64_t T, int32_t G, int32_t nseg, int32_t hq, int64_t max_pairs) {
    DecPlan p{};
    int64_t o = 0;
    p.off_first_seg = o; o = dec_a256(o + 4 * int64_t(G + 1));
    p.off_seg_group = o; o = dec_a256(o + 4 * int64_t(nseg));
    p.off_unit_off = o;  o = dec_a256(o + 4 * int64_t(nseg + 1));
    p.off_pair_off = o;  o = dec_a256(o + 4 * int64_t(nseg + 1));
    p.off_job_off = o;   o = dec_a256(o + 4 * int64_t(nseg + 1));
    p.off_counts = o;    o = dec_a256(o + 16);
    p.off_jobs = o;      o = dec_a256(o + 32 * max_pairs);
    p.off_resp = o;      o = dec_a256(o + 32 * int64_t(nseg - G));
    p.off_part = o;      o = dec_a256(o + 4 * max_pairs * hq * DEC_REC);
    p.total = o;
    p.max_pairs = max_pairs;
    (void)T;
    return p;
}

template <typename T> __device__ __forceinline__ T *dec_ptr(void *ws, int64_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}
template <typename T> __device__ __forceinline__ const T *dec_ptr(const void *ws, int64_t off) {
    return reinterpret_cast<const T *>(static_cast<const char *>(ws) + off);
}

// One job (a 128-key chunk of a segment x a query block), decoded once by the plan kernel so that the roles of the
// chunk kernel read it with one load instead of searching the segment offsets.
struct alignas(16) DecJobRec {
    int32_t y0, yend;    // packed keys [y0, min(y0 + DEC_CH, yend)) of the chunk
    int32_t r0, nq;      // first response of the query block and how many of its responses see the chunk
    int32_t pbase;       // record of (this chunk, the block's first response)
    int32_t pad[3];
};

// Where one response's records lie: its prefix chunks' records are pp0 + j * stride (j < nch_p), its own chunks'
// records po + j (j < nch_o).
struct alignas(16) DecRespRec {
    int32_t pp0, stride, nch_p, po, nch_o;
    int32_t pad[3];
};

// groups: pp_group_desc pairs {prefix_len, num_suffixes}; cu: int32[nseg + 1]. rb = responses per query block.
__global__ void __launch_bounds__(1024) k_dec_plan(const int32_t *__restrict__ groups, int32_t G,
                                                   const int32_t *__restrict__ cu, int32_t nseg, int64_t T, int rb,
                                                   void *ws, DecPlan p) {
    constexpr int NT = 1024;
    __shared__ int32_t s_tmp[3 * 32];
    __shared__ int32_t s_bad;
    int32_t *first_seg = dec_ptr<int32_t>(ws, p.off_first_seg);
    int32_t *seg_group = dec_ptr<int32_t>(ws, p.off_seg_group);
    int32_t *unit_off = dec_ptr<int32_t>(ws, p.off_unit_off);
    int32_t *pair_off = dec_ptr<int32_t>(ws, p.off_pair_off);
    int32_t *job_off = dec_ptr<int32_t>(ws, p.off_job_off);
    int32_t *counts = dec_ptr<int32_t>(ws, p.off_counts);
    if (threadIdx.x == 0) s_bad = (cu[0] != 0 || int64_t(cu[nseg]) != T) ? 1 : 0;
    __syncthreads();
    for (int s = threadIdx.x; s < nseg; s += NT)
        if (cu[s + 1] < cu[s]) s_bad = 1;                      // segment bounds must stay inside [0, T]
    for (int g = threadIdx.x; g < G; g += NT) {
        const int32_t kg = groups[2 * g + 1];
        if (kg < 0) s_bad = 1;
        first_seg[g] = 1 + (kg < 0 ? 0 : kg);
    }
    if (threadIdx.x == 0) first_seg[G] = 0;
    __syncthreads();
    const int32_t tot_seg = block_exclusive_scan<NT>(first_seg, G + 1, s_tmp);
    if (tot_seg != nseg || s_bad) {                            // descriptors disagree with the segments
        if (threadIdx.x == 0) {
            atomicOr(&g_dev_err, DEVERR_BAD_GROUPS);
            counts[0] = 0;
            counts[1] = 0;
            counts[2] = 0;
            counts[3] = 0;
        }
        return;
    }
    for (int g = threadIdx.x; g < G; g += NT)                  // each group labels its own run of segments
        for (int s = first_seg[g]; s < first_seg[g + 1]; ++s) seg_group[s] = g;
    __syncthreads();
    for (int s = threadIdx.x; s < nseg; s += NT) {
        const int g = seg_group[s];
        const int32_t len = cu[s + 1] - cu[s];
        const int32_t nch = len > 0 ? (len + DEC_CH - 1) / DEC_CH : 0;
        const int32_t q_per = (s == first_seg[g]) ? groups[2 * g + 1] : 1;
        unit_off[s] = nch;
        pair_off[s] = nch * q_per;
        job_off[s] = nch * ((q_per + rb - 1) / rb);
    }
    if (threadIdx.x == 0) {
        unit_off[nseg] = 0;
        pair_off[nseg] = 0;
        job_off[nseg] = 0;
    }
    __syncthreads();
    int32_t *const arrs[3] = {unit_off, pair_off, job_off};
    int32_t tots[3];
    block_exclusive_scan_multi<NT, 3>(arrs, nseg + 1, s_tmp, tots);
    const int32_t U = tots[0], NP = tots[1], NJ = tots[2];
    const bool fits = int64_t(NP) <= p.max_pairs;              // the job table (NJ <= NP entries) fits too
    if (fits) {
        DecJobRec *jobs = dec_ptr<DecJobRec>(ws, p.off_jobs);
        DecRespRec *resp_tab = dec_ptr<DecRespRec>(ws, p.off_resp);
        for (int s = threadIdx.x; s < nseg; s += NT) {
            const int g = seg_group[s];
            const int sp = first_seg[g];
            const bool prefix = s == sp;
            const int kg = groups[2 * g + 1];
            const int cnt = prefix ? kg : 1;                   // queries that see the segment
            const int nch = unit_off[s + 1] - unit_off[s];
            const int resp0 = prefix ? sp - g : s - g - 1;     // response ordinal = segment - group - 1
            const int nw = job_off[s + 1] - job_off[s];
            const int y_s = cu[s], y_e = cu[s + 1], pb = pair_off[s], jb = job_off[s];
            for (int w = 0; w < nw; ++w) {                     // (query block, chunk), chunks fastest: one Q load
                const int qb = w / nch, j = w % nch;           // serves all chunks of the segment
                DecJobRec r;
                r.y0 = y_s + j * DEC_CH;
                r.yend = y_e;
                r.r0 = resp0 + qb * rb;
                r.nq = min(rb, cnt - qb * rb);
                r.pbase = pb + j * cnt + qb * rb;
                r.pad[0] = r.pad[1] = r.pad[2] = 0;
                jobs[jb + w] = r;
            }
            if (!prefix) {
                const int i = s - sp - 1;                      // response index within the group
                DecRespRec rr;
                rr.pp0 = pair_off[sp] + i;
                rr.stride = kg;
                rr.nch_p = unit_off[sp + 1] - unit_off[sp];
                rr.po = pb;
                rr.nch_o = nch;
                rr.pad[0] = rr.pad[1] = rr.pad[2] = 0;
                resp_tab[resp0] = rr;
            }
        }
    }
    if (threadIdx.x == 0) {
        if (!fits) atomicOr(&g_dev_err, DEVERR_BAD_GROUPS);   // descriptors differ from the sized ones
        counts[0] = fits ? U : 0;
        counts[1] = NP;
        counts[2] = fits ? 1 : 0;
        counts[3] = fits ? NJ : 0;
    }
}

struct DecSmem {
    static constexpr int TILE = 128 * DEC_D * 2;        // 128 rows x d bf16 (two 64-column 128-byte-swizzled chunks)
    static constexpr int CHUNK = 128 * 64 * 2;
    alignas(1024) uint8_t q[TILE];
    alignas(1024) uint8_t k[DEC_STAGES][TILE];
    alignas(1024) uint8_t v[DEC_STAGES][TILE];
    uint64_t q_full, q_empty;
    uint64_t k_full[DEC_STAGES], k_empty[DEC_STAGES], v_full[DEC_STAGES], v_empty[DEC_STAGES];
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(DecSmem) + 1024 <= 232448, "decode kernel shared memory exceeds 227 KB");

// One job: chunk of one segment, kv head kh, one query block.
struct DecJob {
    int kh;
    int y0, yend;         // packed keys [y0, min(y0 + DEC_CH, yend)) of the chunk
    int r0;               // response ordinal of the block's first query row
    int nq;               // responses of this block that see the chunk (<= rb)
    int64_t pbase;        // record of (this chunk, the block's first response)
};

__device__ __forceinline__ DecJob dec_job(const void *ws, const DecPlan &p, int J, int64_t jj) {
    const DecJobRec r = dec_ptr<DecJobRec>(ws, p.off_jobs)[jj % J];
    DecJob d;
    d.kh = int(jj / J);
    d.y0 = r.y0;
    d.yend = r.yend;
    d.r0 = r.r0;
    d.nq = r.nq;
    d.pbase = r.pbase;
    return d;
}

// q: [n_resp, hq, D] (one query per response, responses in packed order); k, v: [T, hkv, D] cache.
// tmQ: 3-D map over q (d, hq, n_resp) with box (64, r, rb); tmK/tmV: 3-D maps over the cache, box (64, 1, 128).
__global__ void __launch_bounds__(DEC_THREADS, 1)
k_dec_chunk(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
            const __grid_constant__ CUtensorMap tmV, int hq, int hkv, int rb, int32_t n_resp, float sl2, void *ws,
            DecPlan p) {
    extern __shared__ uint8_t smem_raw[];
    DecSmem &sm = *reinterpret_cast<DecSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = hq / hkv;
    volatile int *abort_flag = &sm.abort_flag;
    float *part = dec_ptr<float>(ws, p.off_part);

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_empty, 1);
        for (int s = 0; s < DEC_STAGES; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_full[b], 128);
            mbar_init(&sm.o_full[b], 1);
            mbar_init(&sm.o_free[b], 128);
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
    const int32_t J = dec_ptr<int32_t>(ws, p.off_counts)[3];
    const int64_t n_jobs = int64_t(J) * hkv;
    // contiguous job range per CTA: consecutive jobs share a query block (one Q load per segment and kv head)
    const int64_t j_begin = n_jobs * blockIdx.x / gridDim.x, j_end = n_jobs * (blockIdx.x + 1) / gridDim.x;
    const uint32_t tmem = sm.tmem_base;
    // TMEM: S_b [128 b, 128 b + 128), O_b [256 + 128 b, ...); P_b (bf16) over the first 64 columns of S_b
    auto same_q = [&](const DecJob &a, const DecJob &b) { return a.kh == b.kh && a.r0 == b.r0; };

    if (J == 0) {
        // nothing planned (or the plan did not fit: the combine kernel reports it)
    } else if (warp == 8) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t nq_loads = 0;
            DecJob prev{};
            for (int64_t jj = j_begin; jj < j_end; ++jj) {
                const DecJob d = dec_job(ws, p, J, jj);
                const uint32_t u = uint32_t(jj - j_begin);
                if (u == 0 || !same_q(d, prev)) {
                    if (!bwait(&sm.q_empty, (nq_loads & 1) ^ 1, abort_flag)) break;
                    ++nq_loads;
                    mbar_arrive_expect_tx(&sm.q_full, uint32_t(r * rb) * DEC_D * 2);
                    for (int c = 0; c < DEC_D / 64; ++c)
                        tma_load_3d(sm.q + c * DecSmem::CHUNK, &tmQ, c * 64, d.kh * r, d.r0, &sm.q_full);
                }
                prev = d;
                const int st = u % DEC_STAGES;
                const uint32_t ph = ((u / DEC_STAGES) & 1) ^ 1;
                if (!bwait(&sm.k_empty[st], ph, abort_flag)) break;
                mbar_arrive_expect_tx(&sm.k_full[st], DecSmem::TILE);
                for (int c = 0; c < DEC_D / 64; ++c)
                    tma_load_3d(sm.k[st] + c * DecSmem::CHUNK, &tmK, c * 64, d.kh, d.y0, &sm.k_full[st]);
                if (!bwait(&sm.v_empty[st], ph, abort_flag)) break;
                mbar_arrive_expect_tx(&sm.v_full[st], DecSmem::TILE);
                for (int c = 0; c < DEC_D / 64; ++c)
                    tma_load_3d(sm.v[st] + c * DecSmem::CHUNK, &tmV, c * 64, d.kh, d.y0, &sm.v_full[st]);
            }
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------------ MMA issuer (one thread)
        // Order: S(0), S(1), PV(0), S(2), PV(1), ... S(u + 2) overwrites the columns PV(u) reads, after it in issue
        // order; PV(u) also waits until the record warps have read O of job u - 2 (same buffer).
        if (lane == 0 && j_begin < j_end) {
            constexpr uint32_t ID_S = idesc_bf16(128, DEC_CH, 0, 0);
            constexpr uint32_t ID_O = idesc_bf16(128, DEC_D, 0, 1);
            constexpr uint32_t TB = DecSmem::TILE;
            const uint64_t q_desc = smem_desc(smem_u32(sm.q), 16, 1024);
            const uint64_t k_desc = smem_desc(smem_u32(sm.k[0]), 16, 1024);
            const uint64_t v_desc = smem_desc(smem_u32(sm.v[0]), DecSmem::CHUNK, 1024);
            const uint32_t nu = uint32_t(j_end - j_begin);
            uint32_t nq_used = 0;
            DecJob prev{};
            auto issue_s = [&](uint32_t u) -> bool {
                const DecJob d = dec_job(ws, p, J, j_begin + u);
                if (u == 0 || !same_q(d, prev)) {
                    if (u > 0) umma_commit(&sm.q_empty);                 // the previous block's last S is issued
                    if (!bwait(&sm.q_full, nq_used & 1, abort_flag)) return false;
                    ++nq_used;
                }
                prev = d;
                const int st = u % DEC_STAGES;
                if (!bwait(&sm.k_full[st], (u / DEC_STAGES) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint64_t b = k_desc + uint64_t(st) * (TB >> 4);
                const uint32_t dst = tmem + 128 * (u & 1);
#pragma unroll
                for (int kk = 0; kk < DEC_D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * DecSmem::CHUNK + (kk & 3) * 32;
                    umma_ss(dst, desc_adv(q_desc, off), desc_adv(b, off), ID_S, kk > 0);
                }
                umma_commit(&sm.s_full[u & 1]);
                umma_commit(&sm.k_empty[st]);
                return true;
            };
            bool ok = issue_s(0) && (nu < 2 || issue_s(1));
            for (uint32_t u = 0; ok && u < nu; ++u) {
                const int b = u & 1, st = u % DEC_STAGES;
                if (!bwait(&sm.p_full[b], (u >> 1) & 1, abort_flag)) break;
                if (!bwait(&sm.o_free[b], ((u >> 1) & 1) ^ 1, abort_flag)) break;
                if (!bwait(&sm.v_full[st], (u / DEC_STAGES) & 1, abort_flag)) break;
                tc_fence_after();
                const uint64_t bv = v_desc + uint64_t(st) * (TB >> 4);
#pragma unroll
                for (int kk = 0; kk < DEC_CH / 16; ++kk)
                    umma_ts(tmem + 256 + 128 * b, tmem + 128 * b + kk * 8, desc_adv(bv, kk * 2048), ID_O, kk > 0);
                umma_commit(&sm.o_full[b]);
                umma_commit(&sm.v_empty[st]);
                if (u + 2 < nu) ok = issue_s(u + 2);
            }
            if (ok) umma_commit(&sm.q_empty);
        }
    } else {
        // ------------------------------------------------------------------ softmax and record warpgroups (0-7)
        // Warpgroup b (warps 4b..4b+3) takes the jobs u with u % 2 == b, so it always uses TMEM buffer b, and the
        // two warpgroups' chains (S -> P -> PV -> record) overlap. Thread = query row t of the block (TMEM lane):
        // response r0 + t / r, q head kh * r + t % r. Warps whose rows are all idle skip the TMEM traffic.
        const int b = warp >> 2;
        const int t = threadIdx.x & 127;
        const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
        const int tr = t / r, th = t % r;
        const uint32_t nu = uint32_t(j_end - j_begin);
        for (uint32_t u = b; u < nu; u += 2) {
            const DecJob d = dec_job(ws, p, J, j_begin + u);
            const bool valid = t < r * rb && tr < d.nq && d.r0 + tr < n_resp;
            const int nk = min(DEC_CH, d.yend - d.y0);             // keys of the chunk inside the segment
            if (!bwait(&sm.s_full[b], (u >> 1) & 1, abort_flag)) goto done;
            tc_fence_after();
            float m = -INFINITY, l = 0.f;                          // record: max of S * sl2 (base 2), sum of P
            const bool any = __any_sync(0xffffffffu, valid);
            if (any) {
                // Rows that are not valid are not masked: their P and O are never read.
                float s[DEC_CH];
                {
                    uint32_t r0[32], r1[32], r2[32], r3[32];
                    tmem_ld32(tmem + lane_off + 128 * b, r0);
                    tmem_ld32(tmem + lane_off + 128 * b + 32, r1);
                    tmem_ld32(tmem + lane_off + 128 * b + 64, r2);
                    tmem_ld32(tmem + lane_off + 128 * b + 96, r3);
                    tmem_wait_ld(r0, r1, r2, r3);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        s[e] = __uint_as_float(r0[e]);
                        s[32 + e] = __uint_as_float(r1[e]);
                        s[64 + e] = __uint_as_float(r2[e]);
                        s[96 + e] = __uint_as_float(r3[e]);
                    }
                }
                if (nk < DEC_CH) {                                 // the segment's last chunk: keys past its end
#pragma unroll
                    for (int c = 0; c < DEC_CH; ++c)
                        if (c >= nk) s[c] = -INFINITY;
                }
                float mx = s[0];
#pragma unroll
                for (int c = 1; c + 1 < DEC_CH; c += 2) mx = fmax3(mx, s[c], s[c + 1]);
                mx = fmaxf(mx, s[DEC_CH - 1]);
                // the scale is positive, so max(S) * sl2 is the max of the scaled row; P = 2^(S * sl2 - mu)
                const float mu = mx == -INFINITY ? 0.f : mx * sl2;
                m = mx == -INFINITY ? -INFINITY : mu;
#pragma unroll
                for (int c = 0; c < DEC_CH / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 x = ffma2(make_float2(s[32 * c + 2 * e], s[32 * c + 2 * e + 1]),
                                               make_float2(sl2, sl2), make_float2(-mu, -mu));
                        const float2 pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        l += pp.x + pp.y;
                        pk[e] = pack_bf16x2(pp.x, pp.y);
                    }
                    tmem_st16(tmem + lane_off + 128 * b + 16 * c, pk);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(&sm.p_full[b]);
            // the job's O (PV(u)) -> its record (max in base-2 units, sum, six pad, O[128])
            if (!bwait(&sm.o_full[b], (u >> 1) & 1, abort_flag)) goto done;
            tc_fence_after();
            if (any) {
                const int64_t rec = ((d.pbase + tr) * hq + d.kh * r + th) * int64_t(DEC_REC);
#pragma unroll
                for (int c = 0; c < DEC_D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + 256 + 128 * b + 32 * c, o);
                    tmem_wait_ld(o);
                    if (valid) {
                        float *dst = part + rec + DEC_REC_O + 32 * c;       // 32-byte aligned
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            st_global_32(dst + 8 * e, true, o[8 * e], o[8 * e + 1], o[8 * e + 2], o[8 * e + 3],
                                         o[8 * e + 4], o[8 * e + 5], o[8 * e + 6], o[8 * e + 7]);
                    }
                }
                if (valid) *reinterpret_cast<float4 *>(part + rec) = make_float4(m, l, 0.f, 0.f);
            }
            tc_fence_before();
            mbar_arrive(&sm.o_free[b]);
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

// o: [n_resp, hq, D] bf16; lse: [hq, n_resp] fp32 (natural log).
constexpr int DEC_COMB_WARPS = 8;

// One warp per (response, q head); a lane owns four of the d outputs. The records' maxima are read first (one lane
// per record) to get the common max M; then the records are summed with weights 2^(m - M), eight records' loads in
// flight per lane.
__global__ void __launch_bounds__(DEC_COMB_WARPS * 32, 3) k_dec_combine(int hq, int32_t n_resp, const void *ws,
                                                                     DecPlan p, __nv_bfloat16 *__restrict__ o,
                                                                     float *__restrict__ lse) {
    constexpr int UNROLL = 8;
    const DecRespRec *resp_tab = dec_ptr<DecRespRec>(ws, p.off_resp);
    const float *part = dec_ptr<float>(ws, p.off_part);
    const int32_t ok = dec_ptr<int32_t>(ws, p.off_counts)[2];
    const int lane = threadIdx.x & 31;
    const int64_t n_units = int64_t(n_resp) * hq, stride = int64_t(gridDim.x) * DEC_COMB_WARPS;
    for (int64_t w = int64_t(blockIdx.x) * DEC_COMB_WARPS + (threadIdx.x >> 5); w < n_units; w += stride) {
        const int resp = int(w / hq), hh = int(w % hq);
        __nv_bfloat162 *orow = reinterpret_cast<__nv_bfloat162 *>(o + (int64_t(resp) * hq + hh) * DEC_D + 4 * lane);
        float *lrow = lse + int64_t(hh) * n_resp + resp;
        if (!ok) {                                             // the plan did not fit: no records were written
            const float nan = __int_as_float(0x7fc00000);
            orow[0] = __floats2bfloat162_rn(nan, nan);
            orow[1] = __floats2bfloat162_rn(nan, nan);
            if (lane == 0) *lrow = nan;
            continue;
        }
        const DecRespRec rr = resp_tab[resp];
        const int n = rr.nch_p + rr.nch_o;
        auto rec_of = [&](int j) -> const float * {
            const int64_t pair = j < rr.nch_p ? int64_t(rr.pp0) + int64_t(j) * rr.stride : int64_t(rr.po) + (j - rr.nch_p);
            return part + (pair * hq + hh) * DEC_REC;
        };
        float M = -INFINITY;
        for (int j = lane; j < n; j += 32) M = fmaxf(M, rec_of(j)[0]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        auto add = [&](float m, float l, float4 v) {
            if (m == -INFINITY) return;                        // a chunk with no key visible to this row
            const float wgt = exp2f(m - M);
            L = fmaf(l, wgt, L);
            acc.x = fmaf(v.x, wgt, acc.x);
            acc.y = fmaf(v.y, wgt, acc.y);
            acc.z = fmaf(v.z, wgt, acc.z);
            acc.w = fmaf(v.w, wgt, acc.w);
        };
        if (M != -INFINITY) {
            int j = 0;
            for (; j + UNROLL <= n; j += UNROLL) {
                float m[UNROLL], l[UNROLL];
                float4 v[UNROLL];
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const float *r = rec_of(j + u);
                    m[u] = r[0];
                    l[u] = r[1];
                    v[u] = *reinterpret_cast<const float4 *>(r + DEC_REC_O + 4 * lane);
                }
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) add(m[u], l[u], v[u]);
            }
            for (; j < n; ++j) {
                const float *r = rec_of(j);
                add(r[0], r[1], *reinterpret_cast<const float4 *>(r + DEC_REC_O + 4 * lane));
            }
        }
        const bool any = L > 0.f;
        const float inv = any ? 1.f / L : 0.f;
        orow[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
        orow[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
        if (lane == 0) *lrow = any ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
}

}  // namespace pp
