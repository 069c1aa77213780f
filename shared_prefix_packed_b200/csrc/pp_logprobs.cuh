// pp_logprobs.cuh - log-probabilities of the response tokens, read off the logits of a packed sequence.
//
// What it computes (pp.h, pp_response_logprobs; "prefix_grouper_utils.py" §3, the forward with the grouper): the
// logits are split so that each response's block starts with its group's last prefix row (split_output with
// include_prefix_last=1), each block's last row is dropped, the rows are divided by the temperature, and the
// log-probability of each completion token is read off the log-softmax of its row. On the packed layout the token
// at row y of a response is predicted by row y - 1, except the response's first token, which is predicted by the
// group's last prefix row o_g + P_g - 1. Prefix rows, and a response's first token when P_g = 0, have no
// predicting row and get 0.
//
// HBM-bound: each scored row streams one row of V logits once. One CTA per row at a time (persistent grid); every
// thread keeps an online (max, sum) of 2^(x log2(e) / temperature) over its 16-byte vectors, four loads in flight,
// and the block combines the pairs. The token's own logit is one extra load.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include "pp_meta.cuh"
#include "pp_ptx.cuh"
#include "pp_build.cuh"   // g_dev_err, upper_bound_i32

namespace pp {

constexpr int LP_THREADS = 256;

template <typename T> struct LpVec;
template <> struct LpVec<__nv_bfloat16> {
    static constexpr int N = 8;                                // elements per 16-byte vector
    __device__ static void unpack(const uint4 &u, float (&x)[8]) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static float one(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
};
template <> struct LpVec<float> {
    static constexpr int N = 4;
    __device__ static void unpack(const uint4 &u, float (&x)[4]) {
        x[0] = __uint_as_float(u.x);
        x[1] = __uint_as_float(u.y);
        x[2] = __uint_as_float(u.z);
        x[3] = __uint_as_float(u.w);
    }
    __device__ static float one(const float *p) { return *p; }
};

// Fold the values x (already in base-2 units) into the running (m, s): s = sum 2^(x - m).
template <int N>
__device__ __forceinline__ void lse2_add(float &m, float &s, const float (&x)[N]) {
    float vm = x[0];
#pragma unroll
    for (int i = 1; i < N; ++i) vm = fmaxf(vm, x[i]);
    if (vm == -INFINITY) return;                               // all masked: adds nothing (and -inf - -inf is NaN)
    if (vm > m) {
        s *= ex2_approx(m - vm);                               // m = -inf: s is 0 and stays 0
        m = vm;
    }
#pragma unroll
    for (int i = 0; i < N; ++i) s += ex2_approx(x[i] - m);
}

// Combine two (m, s) pairs.
__device__ __forceinline__ void lse2_merge(float &m, float &s, float om, float os) {
    const float M = fmaxf(m, om);
    if (M == -INFINITY) return;                                // both empty
    s = s * ex2_approx(m - M) + os * ex2_approx(om - M);
    m = M;
}

template <typename T>
__global__ void __launch_bounds__(LP_THREADS) k_response_logprobs(const T *__restrict__ logits, int64_t V,
                                                                  const int32_t *__restrict__ ids,
                                                                  const void *__restrict__ meta, float c2,
                                                                  float inv_temp, float *__restrict__ out) {
    using Vec = LpVec<T>;
    constexpr int N = Vec::N;
    __shared__ float red_m[LP_THREADS / 32], red_s[LP_THREADS / 32];
    const MetaHeader hd = *meta_ptr<MetaHeader>(meta, 0);
    if (hd.dev_err) return;
    const int64_t Tn = hd.T;
    const GroupInfo *groups = meta_ptr<GroupInfo>(meta, hd.off_groups);
    const int32_t *seg_start = meta_ptr<int32_t>(meta, hd.off_seg_start);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t y = blockIdx.x; y < Tn; y += gridDim.x) {
        // the group of row y: the last group whose start is <= y (binary search over the group starts)
        int lo = 0, hi = hd.G;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (groups[mid].start <= y) lo = mid + 1; else hi = mid;
        }
        const GroupInfo gi = groups[lo - 1];
        int64_t src = -1;
        if (y >= int64_t(gi.start) + gi.plen) {                                   // a response row
            if (seg_start[y] == y) src = gi.plen > 0 ? int64_t(gi.start) + gi.plen - 1 : -1;
            else src = y - 1;
        }
        if (src < 0) {
            if (threadIdx.x == 0) out[y] = 0.f;
            continue;
        }
        const int32_t tok = ids[y];
        if (tok < 0 || int64_t(tok) >= V) {
            if (threadIdx.x == 0) {
                out[y] = __int_as_float(0x7fc00000);                              // NaN
                atomicOr(&g_dev_err, DEVERR_BAD_TOKEN);
            }
            continue;
        }
        const T *row = logits + src * V;
        float m = -INFINITY, s = 0.f;
        // scalar head up to the first 16-byte boundary, 16-byte vectors, scalar tail
        const int64_t mis = (reinterpret_cast<uintptr_t>(row) & 15) / sizeof(T);
        const int64_t head = mis ? (16 / int64_t(sizeof(T)) - mis < V ? 16 / int64_t(sizeof(T)) - mis : V) : 0;
        const int64_t nvec = (V - head) / N;
        if (threadIdx.x < head) {
            float x[1] = {Vec::one(row + threadIdx.x) * c2};
            lse2_add<1>(m, s, x);
        }
        const uint4 *vrow = reinterpret_cast<const uint4 *>(row + head);
        int64_t i = threadIdx.x;
        for (; i + 3 * LP_THREADS < nvec; i += 4 * LP_THREADS) {                  // four loads in flight
            uint4 u[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) u[k] = __ldg(vrow + i + k * LP_THREADS);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float x[N];
                Vec::unpack(u[k], x);
#pragma unroll
                for (int e = 0; e < N; ++e) x[e] *= c2;
                lse2_add<N>(m, s, x);
            }
        }
        for (; i < nvec; i += LP_THREADS) {
            float x[N];
            Vec::unpack(__ldg(vrow + i), x);
#pragma unroll
            for (int e = 0; e < N; ++e) x[e] *= c2;
            lse2_add<N>(m, s, x);
        }
        for (int64_t t = head + nvec * N + threadIdx.x; t < V; t += LP_THREADS) {
            float x[1] = {Vec::one(row + t) * c2};
            lse2_add<1>(m, s, x);
        }
        // block reduction of (m, s)
#pragma unroll
        for (int off = 16; off; off >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, m, off);
            const float os = __shfl_xor_sync(0xffffffffu, s, off);
            lse2_merge(m, s, om, os);
        }
        if (lane == 0) {
            red_m[warp] = m;
            red_s[warp] = s;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            float M = red_m[0], S = red_s[0];
            for (int w = 1; w < LP_THREADS / 32; ++w) lse2_merge(M, S, red_m[w], red_s[w]);
            // log p = x_tok / temperature - ln 2 * (M + log2 S)
            out[y] = Vec::one(row + tok) * inv_temp - 0.69314718055994531f * (M + __log2f(S));
        }
        __syncthreads();
    }
}

}  // namespace pp
