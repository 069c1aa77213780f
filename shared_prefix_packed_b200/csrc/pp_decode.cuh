// pp_decode.cuh - decode-time attention over a group-contiguous KV cache (pp.h, pp_decode_attn).
//
// The cache holds, group by group, the prefix's K/V rows and then each response's rows, the newest token of each
// response last ("PackInfer" abstract: group-contiguous KV, so a shared prefix is read once; "Preference Packing":
// responses share the prompt's attention). Each response has one query, its newest token, which attends to the
// group's prefix and to its own rows, under the same mask as the packed prefill.
// Flash-decoding over 64-key chunks of every cache segment:
//   k_dec_plan     one block: segment -> group, chunk counts and (chunk, query) pair offsets (scans).
//   k_dec_partial  persistent grid over (chunk, kv head): loads the chunk's K/V once into shared memory and
//                  computes, for every query that sees the chunk (all responses of the group for a prefix chunk,
//                  one response for a response chunk) and each of the r q heads, the chunk's max, sum and
//                  un-normalised output. A prefix chunk is therefore read from HBM once per group, not per response.
//   k_dec_combine  per (response, q head): merges its partials (the group's prefix chunks, its own chunks).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "pp_build.cuh"   // block_exclusive_scan, upper_bound_i32

namespace pp {

constexpr int DEC_CH = 64;            // keys per chunk
constexpr int DEC_THREADS = 256;
constexpr int DEC_D = 128;            // head dim
constexpr int DEC_MAXQ = 64;          // query vectors (responses x q heads of one kv head) per pass over a chunk
constexpr int DEC_LD = DEC_D + 4;     // padded fp32 row of K and Q in shared memory: 8 lanes of 16 B hit 32 banks
constexpr int DEC_SMEM = (2 * DEC_CH * DEC_LD + DEC_MAXQ * DEC_LD + DEC_MAXQ * DEC_CH) * 4;  // bytes; sV unpadded

// Plan layout in the workspace (int32 sections, sizes from G and nseg).
struct DecPlan {
    int64_t off_first_seg;   // [G + 1] first segment of each group (exclusive scan of 1 + k_g)
    int64_t off_seg_group;   // [nseg]
    int64_t off_unit_off;    // [nseg + 1] chunks before each segment
    int64_t off_pair_off;    // [nseg + 1] (chunk, query) pairs before each segment
    int64_t off_counts;      // [4]: units, pairs, ok (1 if the plan fits), unused
    int64_t off_part;        // fp32 partials: [pairs][hq][DEC_D + 2]
    int64_t total;
    int64_t max_pairs;       // partial records the workspace holds
};

__host__ __device__ inline int64_t dec_a256(int64_t x) { return (x + 255) & ~int64_t(255); }

// Section offsets for a workspace that holds max_pairs (chunk, query) partial records. The exact number of pairs
// is sum over prefixes of nch * k_g plus sum over responses of nch, nch = ceil(len / DEC_CH); the host sizing call
// computes it from host copies of the descriptors.
__host__ inline DecPlan dec_plan_layout(int64_t T, int32_t G, int32_t nseg, int32_t hq, int64_t max_pairs) {
    DecPlan p{};
    int64_t o = 0;
    p.off_first_seg = o; o = dec_a256(o + 4 * int64_t(G + 1));
    p.off_seg_group = o; o = dec_a256(o + 4 * int64_t(nseg));
    p.off_unit_off = o;  o = dec_a256(o + 4 * int64_t(nseg + 1));
    p.off_pair_off = o;  o = dec_a256(o + 4 * int64_t(nseg + 1));
    p.off_counts = o;    o = dec_a256(o + 16);
    p.off_part = o;      o = dec_a256(o + 4 * max_pairs * hq * (DEC_D + 2));
    p.total = o;
    p.max_pairs = max_pairs;
    (void)T;
    return p;
}

template <typename T> __device__ __forceinline__ T *dec_ptr(void *ws, int64_t off) {
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

// groups: pp_group_desc pairs {prefix_len, num_suffixes}; cu: int32[nseg + 1].
__global__ void __launch_bounds__(1024) k_dec_plan(const int32_t *__restrict__ groups, int32_t G,
                                                   const int32_t *__restrict__ cu, int32_t nseg, int64_t T, void *ws,
                                                   DecPlan p) {
    __shared__ int32_t s_tmp[1024];
    __shared__ int32_t s_bad;
    int32_t *first_seg = dec_ptr<int32_t>(ws, p.off_first_seg);
    int32_t *seg_group = dec_ptr<int32_t>(ws, p.off_seg_group);
    int32_t *unit_off = dec_ptr<int32_t>(ws, p.off_unit_off);
    int32_t *pair_off = dec_ptr<int32_t>(ws, p.off_pair_off);
    int32_t *counts = dec_ptr<int32_t>(ws, p.off_counts);
    if (threadIdx.x == 0) s_bad = (cu[0] != 0 || int64_t(cu[nseg]) != T) ? 1 : 0;
    __syncthreads();
    for (int s = threadIdx.x; s < nseg; s += blockDim.x)
        if (cu[s + 1] < cu[s]) s_bad = 1;                      // segment bounds must stay inside [0, T]
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const int32_t kg = groups[2 * g + 1];
        if (kg < 0) s_bad = 1;
        first_seg[g] = 1 + (kg < 0 ? 0 : kg);
    }
    if (threadIdx.x == 0) first_seg[G] = 0;
    __syncthreads();
    const int32_t tot_seg = block_exclusive_scan<1024>(first_seg, G + 1, s_tmp);
    __syncthreads();
    if (tot_seg != nseg || s_bad) {                            // descriptors disagree with the segments
        if (threadIdx.x == 0) {
            atomicOr(&g_dev_err, DEVERR_BAD_GROUPS);
            counts[0] = 0;
            counts[1] = 0;
            counts[2] = 0;
        }
        return;
    }
    for (int s = threadIdx.x; s < nseg; s += blockDim.x) {
        const int g = upper_bound_i32(first_seg, G + 1, s) - 1;   // first_seg[g] <= s < first_seg[g + 1]
        seg_group[s] = g;
        const int32_t len = cu[s + 1] - cu[s];
        const int32_t nch = len > 0 ? (len + DEC_CH - 1) / DEC_CH : 0;
        const int32_t q_per = (s == first_seg[g]) ? groups[2 * g + 1] : 1;
        unit_off[s] = nch;
        pair_off[s] = nch * q_per;
    }
    if (threadIdx.x == 0) {
        unit_off[nseg] = 0;
        pair_off[nseg] = 0;
    }
    __syncthreads();
    const int32_t U = block_exclusive_scan<1024>(unit_off, nseg + 1, s_tmp);
    __syncthreads();
    const int32_t NP = block_exclusive_scan<1024>(pair_off, nseg + 1, s_tmp);
    if (threadIdx.x == 0) {
        const bool fits = int64_t(NP) <= p.max_pairs;
        if (!fits) atomicOr(&g_dev_err, DEVERR_BAD_GROUPS);   // descriptors differ from the sized ones
        counts[0] = fits ? U : 0;
        counts[1] = NP;
        counts[2] = fits ? 1 : 0;
    }
}

// q: [n_resp, hq, D] (one query per response, responses in packed order); k, v: [T, hkv, D] cache.
__global__ void __launch_bounds__(DEC_THREADS) k_dec_partial(const __nv_bfloat16 *__restrict__ q,
                                                             const __nv_bfloat16 *__restrict__ k,
                                                             const __nv_bfloat16 *__restrict__ v,
                                                             const int32_t *__restrict__ groups, int32_t G,
                                                             const int32_t *__restrict__ cu, int32_t nseg, int hq,
                                                             int hkv, float sl2, void *ws, DecPlan p) {
    extern __shared__ float dsm[];
    float *sK = dsm;                                           // [DEC_CH][DEC_LD]
    float *sV = sK + DEC_CH * DEC_LD;                          // [DEC_CH][DEC_D]
    float *sQ = sV + DEC_CH * DEC_LD;                          // [DEC_MAXQ][DEC_LD]
    float *sS = sQ + DEC_MAXQ * DEC_LD;                        // [DEC_MAXQ][DEC_CH]
    __shared__ float s_m[DEC_MAXQ], s_l[DEC_MAXQ];
    const int32_t *first_seg = dec_ptr<int32_t>(ws, p.off_first_seg);
    const int32_t *seg_group = dec_ptr<int32_t>(ws, p.off_seg_group);
    const int32_t *unit_off = dec_ptr<int32_t>(ws, p.off_unit_off);
    const int32_t *pair_off = dec_ptr<int32_t>(ws, p.off_pair_off);
    const int32_t U = dec_ptr<int32_t>(ws, p.off_counts)[0];
    float *part = dec_ptr<float>(ws, p.off_part);
    const int r = hq / hkv;
    for (int64_t w = blockIdx.x; w < int64_t(U) * hkv; w += gridDim.x) {
        const int u = int(w / hkv), kh = int(w % hkv);
        const int s = upper_bound_i32(unit_off, nseg + 1, u) - 1;   // unit_off[s] <= u < unit_off[s + 1]
        const int j = u - unit_off[s];
        const int g = seg_group[s];
        const bool prefix = s == first_seg[g];
        const int k_g = groups[2 * g + 1];
        const int y0 = cu[s] + j * DEC_CH;
        const int n = min(DEC_CH, cu[s + 1] - y0);
        // queries that see this chunk: responses [r0, r0 + cnt) (response ordinal = segment - group - 1)
        const int r0 = prefix ? first_seg[g] - g : s - g - 1;
        const int cnt = prefix ? k_g : 1;
        const int64_t pbase = int64_t(pair_off[s]) + int64_t(j) * cnt;   // pair of (this chunk, query r0)
        // chunk K/V (kv head kh) into shared memory as fp32
        for (int e = threadIdx.x; e < DEC_CH * (DEC_D / 8); e += DEC_THREADS) {
            const int row = e / (DEC_D / 8), c8 = (e % (DEC_D / 8)) * 8;
            float kv[2][8];
            if (row < n) {
                const int64_t off = (int64_t(y0 + row) * hkv + kh) * DEC_D + c8;
                const uint4 uk = *reinterpret_cast<const uint4 *>(k + off);
                const uint4 uv = *reinterpret_cast<const uint4 *>(v + off);
                const uint32_t wk[4] = {uk.x, uk.y, uk.z, uk.w}, wv[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    kv[0][2 * i] = __uint_as_float(wk[i] << 16);
                    kv[0][2 * i + 1] = __uint_as_float(wk[i] & 0xffff0000u);
                    kv[1][2 * i] = __uint_as_float(wv[i] << 16);
                    kv[1][2 * i + 1] = __uint_as_float(wv[i] & 0xffff0000u);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) kv[0][i] = kv[1][i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                sK[row * DEC_LD + c8 + i] = kv[0][i];
                sV[row * DEC_D + c8 + i] = kv[1][i];
            }
        }
        // query vectors in passes of DEC_MAXQ: index t = response (t / r) and q head (kh * r + t % r)
        const int m_all = cnt * r;
        for (int t0 = 0; t0 < m_all; t0 += DEC_MAXQ) {
            const int m = min(DEC_MAXQ, m_all - t0);
            __syncthreads();                                   // sK/sV written; previous pass done with sQ/sS
            for (int e = threadIdx.x; e < m * (DEC_D / 8); e += DEC_THREADS) {
                const int t = e / (DEC_D / 8), c8 = (e % (DEC_D / 8)) * 8;
                const int resp = r0 + (t0 + t) / r, hh = kh * r + (t0 + t) % r;
                const uint4 uq = *reinterpret_cast<const uint4 *>(q + (int64_t(resp) * hq + hh) * DEC_D + c8);
                const uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    sQ[t * DEC_LD + c8 + 2 * i] = __uint_as_float(wq[i] << 16);
                    sQ[t * DEC_LD + c8 + 2 * i + 1] = __uint_as_float(wq[i] & 0xffff0000u);
                }
            }
            __syncthreads();
            // scores in base-2 units: S[t][c] = q_t . k_c * scale * log2(e)
            for (int e = threadIdx.x; e < m * DEC_CH; e += DEC_THREADS) {
                const int t = e / DEC_CH, c = e % DEC_CH;
                float acc = -INFINITY;
                if (c < n) {
                    const float4 *qa = reinterpret_cast<const float4 *>(sQ + t * DEC_LD);
                    const float4 *ka = reinterpret_cast<const float4 *>(sK + c * DEC_LD);
                    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
                    for (int i = 0; i < DEC_D / 4; ++i) {
                        const float4 x = qa[i], y = ka[i];
                        a0 = fmaf(x.x, y.x, a0);
                        a1 = fmaf(x.y, y.y, a1);
                        a2 = fmaf(x.z, y.z, a2);
                        a3 = fmaf(x.w, y.w, a3);
                    }
                    acc = ((a0 + a1) + (a2 + a3)) * sl2;
                }
                sS[t * DEC_CH + c] = acc;
            }
            __syncthreads();
            // per query: max and sum of 2^(S - max); S becomes the probabilities
            for (int t = threadIdx.x; t < m; t += DEC_THREADS) {
                float mx = -INFINITY;
                for (int c = 0; c < n; ++c) mx = fmaxf(mx, sS[t * DEC_CH + c]);
                float l = 0.f;
                for (int c = 0; c < DEC_CH; ++c) {
                    const float pv = c < n ? exp2f(sS[t * DEC_CH + c] - mx) : 0.f;
                    sS[t * DEC_CH + c] = pv;
                    l += pv;
                }
                s_m[t] = mx;
                s_l[t] = l;
            }
            __syncthreads();
            // un-normalised output and the partial record (max in base-2 units, sum, O[D])
            for (int e = threadIdx.x; e < m * DEC_D; e += DEC_THREADS) {
                const int t = e / DEC_D, dd = e % DEC_D;
                float acc = 0.f;
                for (int c = 0; c < n; ++c) acc = fmaf(sS[t * DEC_CH + c], sV[c * DEC_D + dd], acc);
                const int resp_i = (t0 + t) / r, hh = kh * r + (t0 + t) % r;
                float *rec = part + ((pbase + resp_i) * hq + hh) * (DEC_D + 2);
                rec[2 + dd] = acc;
                if (dd == 0) {
                    rec[0] = s_m[t];
                    rec[1] = s_l[t];
                }
            }
        }
        __syncthreads();                                       // before the next chunk overwrites sK/sV
    }
}

// o: [n_resp, hq, D] bf16; lse: [hq, n_resp] fp32 (natural log).
__global__ void __launch_bounds__(DEC_D) k_dec_combine(const int32_t *__restrict__ groups, int32_t G,
                                                       const int32_t *__restrict__ cu, int32_t nseg, int hq,
                                                       int32_t n_resp, const void *ws, DecPlan p,
                                                       __nv_bfloat16 *__restrict__ o, float *__restrict__ lse) {
    const int32_t *first_seg = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + p.off_first_seg);
    const int32_t *unit_off = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + p.off_unit_off);
    const int32_t *pair_off = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + p.off_pair_off);
    const float *part = reinterpret_cast<const float *>(static_cast<const char *>(ws) + p.off_part);
    const int32_t ok = reinterpret_cast<const int32_t *>(static_cast<const char *>(ws) + p.off_counts)[2];
    const int dd = threadIdx.x;
    for (int64_t w = blockIdx.x; w < int64_t(n_resp) * hq; w += gridDim.x) {
        const int resp = int(w / hq), hh = int(w % hq);
        if (!ok) {                                             // the plan did not fit: no partials were written
            o[(int64_t(resp) * hq + hh) * DEC_D + dd] = __float2bfloat16_rn(__int_as_float(0x7fc00000));
            if (dd == 0) lse[int64_t(hh) * n_resp + resp] = __int_as_float(0x7fc00000);
            continue;
        }
        // group of the response: the last g with first_seg[g] - g <= resp (responses before group g)
        int lo = 0, hi = G;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (first_seg[mid] - mid <= resp) lo = mid + 1; else hi = mid;
        }
        const int g = lo - 1;
        const int sp = first_seg[g], k_g = groups[2 * g + 1];
        const int i = resp - (first_seg[g] - g);               // response index within the group
        const int so = sp + 1 + i;                              // its own segment
        float M = -INFINITY, L = 0.f, acc = 0.f;
        auto merge = [&](int64_t pair) {
            const float *rec = part + (pair * hq + hh) * (DEC_D + 2);
            const float m = rec[0];
            if (m == -INFINITY) return;
            const float Mn = fmaxf(M, m);
            const float a = exp2f(M - Mn), b = exp2f(m - Mn);
            L = L * a + rec[1] * b;
            acc = acc * a + rec[2 + dd] * b;
            M = Mn;
        };
        const int nch_p = unit_off[sp + 1] - unit_off[sp];
        for (int j = 0; j < nch_p; ++j) merge(int64_t(pair_off[sp]) + int64_t(j) * k_g + i);
        const int nch_o = unit_off[so + 1] - unit_off[so];
        for (int j = 0; j < nch_o; ++j) merge(int64_t(pair_off[so]) + j);
        const bool any = L > 0.f;
        o[(int64_t(resp) * hq + hh) * DEC_D + dd] = __float2bfloat16_rn(any ? acc / L : 0.f);
        if (dd == 0) lse[int64_t(hh) * n_resp + resp] = any ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
        (void)cu;
        (void)nseg;
    }
}

}  // namespace pp
