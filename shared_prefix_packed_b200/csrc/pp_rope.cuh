// pp_rope.cuh - rotary embedding at the grouped position ids, in place on Q and K (HBM-bound).
//
// "prefix_grouper_utils.py" section 1: every response restarts at position P, so each response is embedded as if
// it directly followed the prefix. Rotate-half form (the pages do not name the variant): for m < d/2,
// w_m = theta^(-2m/d), a = pos * w_m; the pair (x_m, x_{m+d/2}) is rotated by a (by -a for the inverse).
//
// Layout of the work: a block takes ROPE_TOK tokens at a time. The angles of a token are shared by all of its
// Hq + Hkv heads, so they are formed once per token (in fp64, then reduced to fp32 cos/sin) into shared memory;
// every thread then moves 16-byte vectors: 8 elements of the first half and the matching 8 of the second half.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace pp {

constexpr int ROPE_TOK = 4;
constexpr int ROPE_THREADS = 256;

template <typename T> struct RopeVec;
template <> struct RopeVec<__nv_bfloat16> {
    static constexpr int N = 8;     // elements per 16-byte vector
    using V = uint4;
    __device__ static void unpack(const V &v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static V pack(const float (&f)[8]) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&b);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};
template <> struct RopeVec<float> {
    static constexpr int N = 4;
    using V = float4;
    __device__ static void unpack(const V &v, float (&f)[4]) { f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w; }
    __device__ static V pack(const float (&f)[4]) { return make_float4(f[0], f[1], f[2], f[3]); }
};

template <typename T>
__global__ void __launch_bounds__(ROPE_THREADS) k_rope(T *__restrict__ q, T *__restrict__ k,
                                                       const int32_t *__restrict__ pos, int64_t ntok, int hq,
                                                       int hkv, int d, double log2_theta, int inverse) {
    using RV = RopeVec<T>;
    constexpr int N = RV::N;
    __shared__ double s_w[128];                    // w_m = theta^(-2m/d), m < d/2 <= 128
    __shared__ float s_cos[ROPE_TOK][128];
    __shared__ float s_sin[ROPE_TOK][128];
    const int half = d / 2;
    for (int m = threadIdx.x; m < half; m += blockDim.x) s_w[m] = exp2(-(2.0 * m / d) * log2_theta);
    const int vec_per_head = half / N;
    const int nq_units = (q ? hq : 0) * vec_per_head;
    const int units = nq_units + (k ? hkv : 0) * vec_per_head;
    for (int64_t t0 = int64_t(blockIdx.x) * ROPE_TOK; t0 < ntok; t0 += int64_t(gridDim.x) * ROPE_TOK) {
        __syncthreads();   // previous tokens' tables are no longer read; s_w is ready
        for (int e = threadIdx.x; e < ROPE_TOK * half; e += blockDim.x) {
            const int tt = e / half, m = e % half;
            const int64_t t = t0 + tt;
            if (t < ntok) {
                const double a = static_cast<double>(pos[t]) * s_w[m];
                double sn, cs;
                sincos(a, &sn, &cs);
                s_cos[tt][m] = static_cast<float>(cs);
                s_sin[tt][m] = static_cast<float>(inverse ? -sn : sn);
            }
        }
        __syncthreads();
        const int nt = static_cast<int>(ntok - t0 < ROPE_TOK ? ntok - t0 : ROPE_TOK);
        for (int e = threadIdx.x; e < nt * units; e += blockDim.x) {
            const int tt = e / units, u = e % units;
            const int64_t t = t0 + tt;
            T *row;
            int vi;
            if (u < nq_units) {
                row = q + (t * hq + u / vec_per_head) * d;
                vi = u % vec_per_head;
            } else {
                const int uk = u - nq_units;
                row = k + (t * hkv + uk / vec_per_head) * d;
                vi = uk % vec_per_head;
            }
            typename RV::V *p1 = reinterpret_cast<typename RV::V *>(row) + vi;
            typename RV::V *p2 = reinterpret_cast<typename RV::V *>(row + half) + vi;
            float x1[N], x2[N], y1[N], y2[N];
            RV::unpack(*p1, x1);
            RV::unpack(*p2, x2);
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const float c = s_cos[tt][vi * N + i], s = s_sin[tt][vi * N + i];
                y1[i] = fmaf(x1[i], c, -x2[i] * s);
                y2[i] = fmaf(x2[i], c, x1[i] * s);
            }
            *p1 = RV::pack(y1);
            *p2 = RV::pack(y2);
        }
    }
}

}  // namespace pp
