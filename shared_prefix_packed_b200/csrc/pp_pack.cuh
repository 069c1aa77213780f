// pp_pack.cuh - build the packed batch from an ungrouped micro-batch on the device (pp.h, pp_pack_batch).
//
// "prefix_grouper_utils.py" §2 (building the grouper from a micro-batch): consecutive samples with equal uids form
// a group; the group's prefix is the prompt of its first sample; the packed input is, group by group, the prefix's
// valid tokens followed by every sample's valid response tokens. Pad-free output plus the descriptors and segment
// boundaries pp_build_meta takes.
// Three launches:
//   k_pack_count   one block per sample: valid prompt and response tokens (row sums of the masks).
//   k_pack_layout  one block: uid runs -> group index of every sample (scan of the head flags), segment lengths in
//                  packed order (prefix of g = segment g + head(g), response of sample i = segment g(i) + 1 + i),
//                  their scan (cu_seqlens), the descriptors, the counts and each sample's packed offsets.
//   k_pack_gather  one block per sample: stream compaction of its valid tokens (warp ballots) to its offsets.
#pragma once
#include <cuda_runtime.h>
#include "pp_build.cuh"   // block_exclusive_scan

namespace pp {

constexpr int PACK_THREADS = 256;
constexpr int PACK_LAYOUT_THREADS = 1024;
constexpr int PACK_MAX_BATCH = 8192;   // samples per micro-batch (the layout block keeps four int32 per sample)

__device__ __forceinline__ int32_t block_sum(int32_t v, int32_t *s_red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    int32_t t = 0;
    if (threadIdx.x == 0)
        for (int w = 0; w < int(blockDim.x >> 5); ++w) t += s_red[w];
    __syncthreads();
    return t;                                                   // valid in thread 0
}

__global__ void __launch_bounds__(PACK_THREADS) k_pack_count(const uint8_t *__restrict__ pm, int32_t Lp,
                                                             const uint8_t *__restrict__ rm, int32_t Lr,
                                                             int32_t *__restrict__ offsets) {
    __shared__ int32_t s_red[PACK_THREADS / 32];
    const int64_t i = blockIdx.x;
    int32_t a = 0, b = 0;
    for (int j = threadIdx.x; j < Lp; j += PACK_THREADS) a += pm[i * Lp + j] != 0;
    for (int j = threadIdx.x; j < Lr; j += PACK_THREADS) b += rm[i * Lr + j] != 0;
    a = block_sum(a, s_red);
    b = block_sum(b, s_red);
    if (threadIdx.x == 0) {
        offsets[2 * i] = a;
        offsets[2 * i + 1] = b;
    }
}

__global__ void __launch_bounds__(PACK_LAYOUT_THREADS) k_pack_layout(const int64_t *__restrict__ uids, int32_t bs,
                                                                     int32_t *__restrict__ offsets,
                                                                     int32_t *__restrict__ groups,
                                                                     int32_t *__restrict__ cu,
                                                                     int32_t *__restrict__ counts) {
    extern __shared__ int32_t sh[];
    int32_t *plen = sh, *rlen = sh + bs, *gid = sh + 2 * bs, *head_of = sh + 3 * bs;
    __shared__ int32_t s_tmp[PACK_LAYOUT_THREADS];
    for (int i = threadIdx.x; i < bs; i += PACK_LAYOUT_THREADS) {
        plen[i] = offsets[2 * i];
        rlen[i] = offsets[2 * i + 1];
        gid[i] = (i == 0 || uids[i] != uids[i - 1]) ? 1 : 0;   // head flag
    }
    __syncthreads();
    const int32_t G = block_exclusive_scan<PACK_LAYOUT_THREADS>(gid, bs, s_tmp);   // heads before i
    for (int i = threadIdx.x; i < bs; i += PACK_LAYOUT_THREADS) {
        const bool head = i == 0 || uids[i] != uids[i - 1];
        gid[i] = gid[i] + (head ? 1 : 0) - 1;                  // group index of sample i
        if (head) head_of[gid[i]] = i;
    }
    __syncthreads();
    const int32_t nseg = G + bs;
    for (int i = threadIdx.x; i < bs; i += PACK_LAYOUT_THREADS) {
        const int g = gid[i];
        if (head_of[g] == i) cu[g + i] = plen[i];             // the group's prefix segment
        cu[g + 1 + i] = rlen[i];                               // sample i's response segment
    }
    if (threadIdx.x == 0) cu[nseg] = 0;
    __syncthreads();
    const int32_t T = block_exclusive_scan<PACK_LAYOUT_THREADS>(cu, nseg + 1, s_tmp);
    (void)T;
    __syncthreads();
    for (int g = threadIdx.x; g < G; g += PACK_LAYOUT_THREADS) {
        const int h = head_of[g];
        const int next = g + 1 < G ? head_of[g + 1] : bs;
        groups[2 * g] = plen[h];                               // pp_group_desc {prefix_len, num_suffixes}
        groups[2 * g + 1] = next - h;
    }
    for (int i = threadIdx.x; i < bs; i += PACK_LAYOUT_THREADS) {
        const int g = gid[i];
        offsets[2 * i] = head_of[g] == i ? cu[g + i] : -1;
        offsets[2 * i + 1] = cu[g + 1 + i];
    }
    if (threadIdx.x == 0) {
        counts[0] = G;
        counts[1] = nseg;
        counts[2] = cu[nseg];
    }
}

// Stream compaction of one masked row into dst[0..): tiles of PACK_THREADS positions, warp ballots for the ranks.
__device__ __forceinline__ void pack_row(const int32_t *__restrict__ tok, const uint8_t *__restrict__ mask, int32_t L,
                                         int32_t *__restrict__ dst, int32_t *s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t base = 0;
    for (int j0 = 0; j0 < L; j0 += PACK_THREADS) {
        const int j = j0 + threadIdx.x;
        const bool on = j < L && mask[j] != 0;
        const uint32_t ball = __ballot_sync(0xffffffffu, on);
        if (lane == 0) s_warp[warp] = __popc(ball);
        __syncthreads();
        int32_t before = 0, total = 0;
        for (int w = 0; w < PACK_THREADS / 32; ++w) {
            const int32_t c = s_warp[w];
            before += w < warp ? c : 0;
            total += c;
        }
        if (on) dst[base + before + __popc(ball & ((1u << lane) - 1u))] = tok[j];
        base += total;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(PACK_THREADS) k_pack_gather(const int32_t *__restrict__ prompts,
                                                              const uint8_t *__restrict__ pm, int32_t Lp,
                                                              const int32_t *__restrict__ responses,
                                                              const uint8_t *__restrict__ rm, int32_t Lr,
                                                              const int32_t *__restrict__ offsets,
                                                              int32_t *__restrict__ packed) {
    __shared__ int32_t s_warp[PACK_THREADS / 32];
    const int64_t i = blockIdx.x;
    const int32_t op = offsets[2 * i], orr = offsets[2 * i + 1];
    if (op >= 0) pack_row(prompts + i * Lp, pm + i * Lp, Lp, packed + op, s_warp);
    pack_row(responses + i * Lr, rm + i * Lr, Lr, packed + orr, s_warp);
}

}  // namespace pp
