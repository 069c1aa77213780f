// pp_api.cu - the C ABI of libpp (declared in include/pp.h): host-side validation, tensor maps, launches, and the
// device error channel. The whole library is this one translation unit; the kernels live in the included headers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/pp.h"
#include "pp_ptx.cuh"
#include "pp_meta.cuh"
#include "pp_build.cuh"
#include "pp_rope.cuh"
#include "pp_attn_fwd.cuh"
#include "pp_attn_bwd.cuh"
#include "pp_logprobs.cuh"
#include "pp_pack.cuh"
#include "pp_decode.cuh"

namespace {

thread_local std::string g_last_error;

pp_status fail(pp_status st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
pp_status fail(pp_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

#define PP_CUDA(call)                                                                                   \
    do {                                                                                                \
        cudaError_t e_ = (call);                                                                        \
        if (e_ != cudaSuccess)                                                                          \
            return fail(PP_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_));                  \
    } while (0)

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

constexpr int kMaxDevices = 64;
struct DeviceInfo {
    bool ready = false;
    int sm_count = 0;
    int max_smem_optin = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

pp_status device_info(DeviceInfo **out) {
    int dev = 0;
    PP_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(PP_ERR_CUDA, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        PP_CUDA(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev));
        PP_CUDA(cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
        int major = 0, minor = 0;
        PP_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
        PP_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
        if (major != 10 || minor != 0)
            return fail(PP_ERR_UNSUPPORTED, "libpp is built for sm_100a (B200); device %d is sm_%d%d", dev, major,
                        minor);
        d.ready = true;
    }
    *out = &d;
    return PP_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time dependency on libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

pp_status get_encoder(EncodeTiledFn *fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(PP_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
        g_encode = reinterpret_cast<EncodeTiledFn>(p);
    }
    *fn = g_encode;
    return PP_OK;
}

// 3-D map over a [rows, heads, d] bf16 tensor: box = 64 elements x box_heads heads x box_rows rows, 128-byte swizzle.
pp_status make_map_3d_box(CUtensorMap *m, const void *base, int64_t rows, int heads, int d, int box_heads,
                          int box_rows);

pp_status make_map_3d(CUtensorMap *m, const void *base, int64_t rows, int heads, int d, int box_rows) {
    return make_map_3d_box(m, base, rows, heads, d, 1, box_rows);
}

pp_status make_map_3d_box(CUtensorMap *m, const void *base, int64_t rows, int heads, int d, int box_heads,
                          int box_rows) {
    EncodeTiledFn enc;
    pp_status st = get_encoder(&enc);
    if (st != PP_OK) return st;
    if (reinterpret_cast<uintptr_t>(base) % 16) return fail(PP_ERR_INVALID_ARG, "tensor base not 16-byte aligned");
    cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(heads), cuuint64_t(rows)};
    cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(heads) * d * 2};
    cuuint32_t box[3] = {64, cuuint32_t(box_heads), cuuint32_t(box_rows)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PP_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
    return PP_OK;
}

pp_status check_heads(int64_t T, int32_t hq, int32_t hkv, int32_t d) {
    if (T < 0 || T >= (int64_t(1) << 31) - 256) return fail(PP_ERR_INVALID_ARG, "T=%lld out of range", (long long)T);
    if (hq <= 0 || hkv <= 0 || hq > 256 || hq % hkv != 0)
        return fail(PP_ERR_INVALID_ARG, "need 0 < hkv, hq %% hkv == 0, hq <= 256 (hq=%d hkv=%d)", hq, hkv);
    if (d != 64 && d != 128) return fail(PP_ERR_INVALID_ARG, "head dim %d not in {64, 128}", d);
    return PP_OK;
}

int grid_for(int sm_count, int per_sm, int64_t work) {
    int64_t g = int64_t(sm_count) * per_sm;
    if (work < g) g = work;
    return int(g < 1 ? 1 : g);
}

// Scratch of pp_attn_bwd_noalloc (see include/pp.h): compiled into the library so that callers who cannot
// allocate still get a backward. Host code must not use the symbol's host-side name as a device address; the
// device address is looked up once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PP_NOALLOC_SCRATCH_BYTES];
void *g_noalloc_ptr[kMaxDevices] = {};

pp_status noalloc_scratch(void **out) {
    int dev = 0;
    PP_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(PP_ERR_CUDA, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);   // with `dev` current
        if (e != cudaSuccess || !p)
            return fail(PP_ERR_CUDA, "cudaGetSymbolAddress(noalloc scratch): %s", cudaGetErrorString(e));
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return PP_OK;
}

}  // namespace

// =====================================================================================================================
extern "C" {

const char *pp_last_error(void) { return g_last_error.c_str(); }

const char *pp_version(void) { return "libpp 0.1 (sm_100a)"; }

pp_status pp_meta_bounds(int32_t num_groups, int32_t num_segments, int64_t total_tokens, int32_t num_heads_q,
                         int32_t num_heads_kv, int64_t *meta_bytes) {
    if (!meta_bytes) return fail(PP_ERR_INVALID_ARG, "meta_bytes is NULL");
    if (num_groups < 1) return fail(PP_ERR_INVALID_ARG, "num_groups must be >= 1");
    if (num_segments < num_groups) return fail(PP_ERR_INVALID_ARG, "num_segments < num_groups");
    pp_status st = check_heads(total_tokens, num_heads_q, num_heads_kv, 128);
    if (st != PP_OK) return st;
    *meta_bytes = pp::meta_layout(total_tokens, num_groups, num_segments, num_heads_q, num_heads_kv).total_bytes;
    return PP_OK;
}

pp_status pp_build_meta(const pp_group_desc *groups_d, int32_t num_groups, const int32_t *cu_seqlens_d,
                        int32_t num_segments, int64_t total_tokens, int32_t num_heads_q, int32_t num_heads_kv,
                        int32_t *pos_ids_d, void *meta_d, int64_t meta_bytes, void *stream) {
    int64_t need = 0;
    pp_status st = pp_meta_bounds(num_groups, num_segments, total_tokens, num_heads_q, num_heads_kv, &need);
    if (st != PP_OK) return st;
    if (!groups_d || !cu_seqlens_d || !meta_d || (total_tokens > 0 && !pos_ids_d))
        return fail(PP_ERR_INVALID_ARG, "NULL device pointer");
    if (reinterpret_cast<uintptr_t>(meta_d) % 256) return fail(PP_ERR_INVALID_ARG, "meta_d not 256-byte aligned");
    if (meta_bytes < need)
        return fail(PP_ERR_WORKSPACE, "meta buffer %lld bytes < %lld needed", (long long)meta_bytes, (long long)need);
    DeviceInfo *di;
    if ((st = device_info(&di)) != PP_OK) return st;
    cudaStream_t s = as_stream(stream);
    const pp::MetaHeader h = pp::meta_layout(total_tokens, num_groups, num_segments, num_heads_q, num_heads_kv);
    pp::k_meta_header<<<1, 1, 0, s>>>(meta_d, h);
    PP_CUDA(cudaGetLastError());
    char *base = reinterpret_cast<char *>(meta_d);
    int32_t *qoff = reinterpret_cast<int32_t *>(base + h.off_scratch);
    int32_t *koff = qoff + (num_groups + 1);
    int32_t *tmp = koff + (num_groups + 1);
    pp::BWork *bw_tmp = reinterpret_cast<pp::BWork *>(base + h.off_bw_tmp);
    pp::k_meta_groups<1024><<<1, 1024, 0, s>>>(groups_d, cu_seqlens_d, meta_d, qoff, koff);
    PP_CUDA(cudaGetLastError());
    if (total_tokens > 0) {
        pp::k_meta_tokens<<<grid_for(di->sm_count, 4, (total_tokens + 255) / 256), 256, 0, s>>>(cu_seqlens_d, meta_d,
                                                                                                  pos_ids_d);
        PP_CUDA(cudaGetLastError());
    }
    const int64_t ntiles = h.cap_qt > h.cap_kt ? h.cap_qt : h.cap_kt;
    pp::k_meta_tiles<<<grid_for(di->sm_count, 2, (ntiles + 127) / 128), 128, 0, s>>>(meta_d, qoff, koff);
    PP_CUDA(cudaGetLastError());
    pp::k_meta_sort<1024><<<1, 1024, 0, s>>>(meta_d, tmp, bw_tmp);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_meta_tiles(const void *meta_d, int32_t which, int32_t *tiles_d, int64_t capacity, int32_t *count_d,
                        void *stream) {
    if (!meta_d || !count_d || (capacity > 0 && !tiles_d)) return fail(PP_ERR_INVALID_ARG, "NULL pointer");
    if (which != PP_PASS_FWD && which != PP_PASS_BWD) return fail(PP_ERR_INVALID_ARG, "which must be fwd or bwd");
    DeviceInfo *di;
    pp_status st = device_info(&di);
    if (st != PP_OK) return st;
    cudaStream_t s = as_stream(stream);
    PP_CUDA(cudaMemsetAsync(count_d, 0, sizeof(int32_t), s));
    pp::k_meta_expand<<<di->sm_count, 128, 0, s>>>(meta_d, which, tiles_d, capacity, count_d);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_meta_schedule(const void *meta_d, int32_t which, int32_t *records_d, int64_t capacity, int32_t *count_d,
                           void *stream) {
    if (!meta_d || !count_d || (capacity > 0 && !records_d)) return fail(PP_ERR_INVALID_ARG, "NULL pointer");
    if (which != PP_PASS_FWD && which != PP_PASS_BWD) return fail(PP_ERR_INVALID_ARG, "which must be fwd or bwd");
    DeviceInfo *di;
    pp_status st = device_info(&di);
    if (st != PP_OK) return st;
    cudaStream_t s = as_stream(stream);
    PP_CUDA(cudaMemsetAsync(count_d, 0, sizeof(int32_t), s));
    pp::k_meta_schedule<<<di->sm_count, 128, 0, s>>>(meta_d, which, records_d, capacity, count_d);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_rope(void *q, void *k, const int32_t *pos_ids_d, int64_t T, int32_t hq, int32_t hkv, int32_t d,
                  float theta, pp_dtype dt, int32_t inverse, void *stream) {
    pp_status st = check_heads(T, hq, hkv, d);
    if (st != PP_OK) return st;
    if (dt != PP_BF16 && dt != PP_FP32) return fail(PP_ERR_INVALID_ARG, "unknown dtype %d", int(dt));
    if (!(theta >= 0.f) || std::isinf(theta)) return fail(PP_ERR_INVALID_ARG, "theta must be finite and >= 0");
    if (T == 0 || (!q && !k)) return PP_OK;
    if (!pos_ids_d) return fail(PP_ERR_INVALID_ARG, "pos_ids_d is NULL");
    if ((q && reinterpret_cast<uintptr_t>(q) % 16) || (k && reinterpret_cast<uintptr_t>(k) % 16))
        return fail(PP_ERR_INVALID_ARG, "q/k must be 16-byte aligned");
    DeviceInfo *di;
    if ((st = device_info(&di)) != PP_OK) return st;
    const double th = theta == 0.f ? 10000.0 : double(theta);
    const int grid = grid_for(di->sm_count, 8, (T + pp::ROPE_TOK - 1) / pp::ROPE_TOK);
    cudaStream_t s = as_stream(stream);
    if (dt == PP_BF16)
        pp::k_rope<__nv_bfloat16><<<grid, pp::ROPE_THREADS, 0, s>>>(
            static_cast<__nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(k), pos_ids_d, T, hq, hkv, d, std::log2(th),
            inverse);
    else
        pp::k_rope<float><<<grid, pp::ROPE_THREADS, 0, s>>>(static_cast<float *>(q), static_cast<float *>(k),
                                                             pos_ids_d, T, hq, hkv, d, std::log2(th), inverse);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_workspace_bytes(int32_t which, int64_t T, int32_t hq, int32_t hkv, int32_t d, int64_t *bytes) {
    if (!bytes) return fail(PP_ERR_INVALID_ARG, "bytes is NULL");
    pp_status st = check_heads(T, hq, hkv, d);
    if (st != PP_OK) return st;
    if (which == PP_PASS_FWD) {
        *bytes = 256;
    } else if (which == PP_PASS_BWD) {
        *bytes = pp::bwd_workspace_layout(T, hq, hkv, d).total;
    } else {
        return fail(PP_ERR_INVALID_ARG, "which must be fwd or bwd");
    }
    return PP_OK;
}

pp_status pp_bwd_ds_bytes(const pp_group_desc *groups_host, int32_t G, const int32_t *cu_host, int32_t nseg,
                          int32_t hq, int32_t hkv, int64_t *bytes) {
    if (!groups_host || !cu_host || !bytes) return fail(PP_ERR_INVALID_ARG, "NULL pointer argument");
    if (G < 0 || nseg < 0 || hq <= 0 || hkv <= 0 || hq % hkv != 0)
        return fail(PP_ERR_INVALID_ARG, "need G, num_segments >= 0 and hq a multiple of hkv");
    const int64_t r = hq / hkv;
    // one step per (key tile, attending query tile, q head): key tile b of a group of length L, prefix P, covers
    // keys [128 b, 128 b + 128); its queries run from its own first row to e = L for a prefix tile, else to the end
    // of the segment of its last key (the same rule as the schedule builder's)
    int64_t steps = 0;
    int32_t s = 0;
    for (int32_t g = 0; g < G; ++g) {
        const int32_t P = groups_host[g].prefix_len, k = groups_host[g].num_suffixes;
        if (k < 0 || P < 0 || s + 1 + int64_t(k) > nseg) return fail(PP_ERR_INVALID_ARG, "descriptors exceed num_segments");
        for (int32_t j = s; j <= s + k; ++j)
            if (cu_host[j + 1] < cu_host[j]) return fail(PP_ERR_INVALID_ARG, "segment bounds must not decrease");
        const int32_t start = cu_host[s], end = cu_host[s + 1 + k];
        const int32_t L = end - start;
        if (cu_host[s + 1] - start != P) return fail(PP_ERR_INVALID_ARG, "prefix length disagrees with segments");
        int32_t seg = s + 1;                                        // segment of the current key (responses)
        for (int32_t y0 = 0; y0 < L; y0 += pp::BWD_BN) {
            const int32_t ylast = std::min(y0 + pp::BWD_BN, L) - 1;
            int32_t e = L;
            if (y0 >= P) {
                while (seg < s + 1 + k && cu_host[seg + 1] - start <= ylast) ++seg;
                e = cu_host[seg + 1] - start;
            }
            const int64_t qa = y0 / pp::BWD_BM, qb = (e + pp::BWD_BM - 1) / pp::BWD_BM;
            steps += (qb - qa) * r * hkv;                          // every q head of every kv head
        }
        s += 1 + k;
    }
    if (s != nseg) return fail(PP_ERR_INVALID_ARG, "num_segments must equal sum_g (1 + k_g)");
    *bytes = pp::BWD_DS_ALIGN + steps * pp::BWD_DS_TILE_BYTES;
    return PP_OK;
}

// Exact (chunk, query) pair count of the decode plan, from host copies of the descriptors and segment bounds.
static pp_status decode_pairs(const pp_group_desc *groups, int32_t G, const int32_t *cu, int32_t nseg, int64_t *pairs) {
    int64_t np = 0;
    int32_t s = 0;
    auto nch = [&](int32_t seg) -> int64_t {
        const int64_t len = int64_t(cu[seg + 1]) - cu[seg];
        return len > 0 ? (len + pp::DEC_CH - 1) / pp::DEC_CH : 0;
    };
    for (int32_t g = 0; g < G; ++g) {
        const int32_t k = groups[g].num_suffixes;
        if (k < 0 || s + 1 + int64_t(k) > nseg) return fail(PP_ERR_INVALID_ARG, "descriptors exceed num_segments");
        np += nch(s) * k;
        for (int32_t i = 0; i < k; ++i) np += nch(s + 1 + i);
        s += 1 + k;
    }
    if (s != nseg) return fail(PP_ERR_INVALID_ARG, "num_segments must equal sum_g (1 + k_g)");
    *pairs = np;
    return PP_OK;
}

pp_status pp_decode_workspace_bytes(const pp_group_desc *groups_host, int32_t G, const int32_t *cu_host, int32_t nseg,
                                    int32_t hq, int64_t *bytes) {
    if (!groups_host || !cu_host || !bytes) return fail(PP_ERR_INVALID_ARG, "NULL pointer argument");
    if (G < 1 || nseg < G || hq < 1) return fail(PP_ERR_INVALID_ARG, "need G >= 1, num_segments >= G, hq >= 1");
    int64_t np;
    pp_status st = decode_pairs(groups_host, G, cu_host, nseg, &np);
    if (st != PP_OK) return st;
    *bytes = pp::dec_plan_layout(cu_host[nseg], G, nseg, hq, np).total;
    return PP_OK;
}

pp_status pp_decode_attn(const void *q, const void *k_cache, const void *v_cache, const pp_group_desc *groups_d,
                         int32_t G, const int32_t *cu_d, int32_t nseg, int64_t T, int32_t hq, int32_t hkv, int32_t d,
                         float softmax_scale, void *o, float *lse, void *workspace, int64_t ws_bytes, void *stream) {
    pp_status st = check_heads(T, hq, hkv, d);
    if (st != PP_OK) return st;
    if (d != pp::DEC_D) return fail(PP_ERR_UNSUPPORTED, "decode supports head dim 128 only (got %d)", d);
    if (G < 1 || nseg < G) return fail(PP_ERR_INVALID_ARG, "need G >= 1 and num_segments >= G");
    const int32_t n_resp = nseg - G;
    if (n_resp == 0) return PP_OK;
    if (!q || !k_cache || !v_cache || !groups_d || !cu_d || !o || !lse || !workspace)
        return fail(PP_ERR_INVALID_ARG, "NULL pointer argument");
    const void *ptrs[4] = {q, k_cache, v_cache, o};
    for (const void *ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) % 16) return fail(PP_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(PP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (!(softmax_scale >= 0.f) || std::isinf(softmax_scale)) return fail(PP_ERR_INVALID_ARG, "bad softmax_scale");
    const int r = hq / hkv;
    if (r > 128) return fail(PP_ERR_UNSUPPORTED, "decode supports at most 128 q heads per kv head (got %d)", r);
    const int rb = 128 / r;                                  // responses per query block (r * rb <= 128 rows)
    const pp::DecPlan base = pp::dec_plan_layout(T, G, nseg, hq, 0);
    const int64_t rec = 4 * int64_t(hq) * pp::DEC_REC + 32;   // one record per q head, and one job entry
    if (ws_bytes < base.total + rec) return fail(PP_ERR_WORKSPACE, "workspace too small for the decode plan");
    int64_t mp = (ws_bytes - base.total) / rec;               // upper bound; trimmed for the sections' alignment
    while (mp > 0 && pp::dec_plan_layout(T, G, nseg, hq, mp).total > ws_bytes) --mp;
    const pp::DecPlan p = pp::dec_plan_layout(T, G, nseg, hq, mp);
    DeviceInfo *di;
    if ((st = device_info(&di)) != PP_OK) return st;
    CUtensorMap mq, mk, mv;
    if ((st = make_map_3d_box(&mq, q, n_resp, hq, d, r, rb)) != PP_OK) return st;
    if ((st = make_map_3d(&mk, k_cache, T, hkv, d, pp::DEC_CH)) != PP_OK) return st;
    if ((st = make_map_3d(&mv, v_cache, T, hkv, d, pp::DEC_CH)) != PP_OK) return st;
    const float scale = softmax_scale == 0.f ? 1.f / std::sqrt(float(d)) : softmax_scale;
    cudaStream_t s = as_stream(stream);
    const int32_t *gd = reinterpret_cast<const int32_t *>(groups_d);
    pp::k_dec_plan<<<1, 1024, 0, s>>>(gd, G, cu_d, nseg, T, rb, workspace, p);
    PP_CUDA(cudaGetLastError());
    const int smem = int(sizeof(pp::DecSmem)) + 1024;
    PP_CUDA(cudaFuncSetAttribute(pp::k_dec_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    pp::k_dec_chunk<<<di->sm_count, pp::DEC_THREADS, smem, s>>>(mq, mk, mv, hq, hkv, rb, n_resp,
                                                                  scale * 1.4426950408889634f, workspace, p);
    PP_CUDA(cudaGetLastError());
    pp::k_dec_combine<<<grid_for(di->sm_count, 3, (int64_t(n_resp) * hq + pp::DEC_COMB_WARPS - 1) / pp::DEC_COMB_WARPS),
                        pp::DEC_COMB_WARPS * 32, 0, s>>>(hq, n_resp, workspace, p, static_cast<__nv_bfloat16 *>(o), lse);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_pack_batch(const int32_t *prompts, const uint8_t *prompt_mask, int32_t Lp, const int32_t *responses,
                        const uint8_t *response_mask, int32_t Lr, const int64_t *uids, int32_t bs,
                        int32_t *packed_ids, int64_t capacity, pp_group_desc *groups, int32_t *cu_seqlens,
                        int32_t *sample_offsets, int32_t *counts, void *stream) {
    if (bs < 0 || bs > pp::PACK_MAX_BATCH)
        return fail(bs < 0 ? PP_ERR_INVALID_ARG : PP_ERR_UNSUPPORTED, "bs must be in [0, %d] (got %d)",
                    pp::PACK_MAX_BATCH, bs);
    if (Lp < 0 || Lr < 0) return fail(PP_ERR_INVALID_ARG, "negative row length");
    const int64_t worst = int64_t(bs) * (int64_t(Lp) + Lr);
    if (worst >= (int64_t(1) << 31)) return fail(PP_ERR_INVALID_ARG, "bs * (Lp + Lr) must fit int32");
    if (capacity < worst) return fail(PP_ERR_INVALID_ARG, "packed_ids capacity %lld < bs * (Lp + Lr) = %lld",
                                      (long long)capacity, (long long)worst);
    if (!cu_seqlens || !counts) return fail(PP_ERR_INVALID_ARG, "NULL pointer argument");
    cudaStream_t s = as_stream(stream);
    if (bs == 0) {
        PP_CUDA(cudaMemsetAsync(counts, 0, 3 * sizeof(int32_t), s));
        PP_CUDA(cudaMemsetAsync(cu_seqlens, 0, sizeof(int32_t), s));
        return PP_OK;
    }
    if (!uids || !groups || !sample_offsets || (worst > 0 && !packed_ids) || (Lp > 0 && (!prompts || !prompt_mask)) ||
        (Lr > 0 && (!responses || !response_mask)))
        return fail(PP_ERR_INVALID_ARG, "NULL pointer argument");
    DeviceInfo *di;
    pp_status st;
    if ((st = device_info(&di)) != PP_OK) return st;
    pp::k_pack_count<<<bs, pp::PACK_THREADS, 0, s>>>(prompt_mask, Lp, response_mask, Lr, sample_offsets);
    PP_CUDA(cudaGetLastError());
    const int smem = 4 * bs * int(sizeof(int32_t));
    PP_CUDA(cudaFuncSetAttribute(pp::k_pack_layout, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    pp::k_pack_layout<<<1, pp::PACK_LAYOUT_THREADS, smem, s>>>(uids, bs, sample_offsets,
                                                               reinterpret_cast<int32_t *>(groups), cu_seqlens,
                                                               counts);
    PP_CUDA(cudaGetLastError());
    pp::k_pack_gather<<<bs, pp::PACK_THREADS, 0, s>>>(prompts, prompt_mask, Lp, responses, response_mask, Lr,
                                                      sample_offsets, packed_ids);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_response_logprobs(const void *logits, pp_dtype dt, int64_t V, const int32_t *token_ids,
                               const void *meta_d, int64_t T, float temperature, float *out, void *stream) {
    if (T < 0 || T >= (int64_t(1) << 31)) return fail(PP_ERR_INVALID_ARG, "T out of range (%lld)", (long long)T);
    if (V < 1) return fail(PP_ERR_INVALID_ARG, "V must be >= 1 (got %lld)", (long long)V);
    if (dt != PP_BF16 && dt != PP_FP32) return fail(PP_ERR_INVALID_ARG, "unknown dtype %d", int(dt));
    if (!(temperature > 0.f) || std::isinf(temperature))
        return fail(PP_ERR_INVALID_ARG, "temperature must be finite and > 0");
    if (T == 0) return PP_OK;
    if (!logits || !token_ids || !meta_d || !out) return fail(PP_ERR_INVALID_ARG, "NULL pointer argument");
    if (reinterpret_cast<uintptr_t>(logits) % (dt == PP_BF16 ? 2 : 4))
        return fail(PP_ERR_INVALID_ARG, "logits must be aligned to their element size");
    DeviceInfo *di;
    pp_status st;
    if ((st = device_info(&di)) != PP_OK) return st;
    const int grid = grid_for(di->sm_count, 8, T);
    const float inv_temp = 1.f / temperature;
    const float c2 = float(1.4426950408889634 / double(temperature));
    cudaStream_t s = as_stream(stream);
    if (dt == PP_BF16)
        pp::k_response_logprobs<__nv_bfloat16><<<grid, pp::LP_THREADS, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(logits), V, token_ids, meta_d, c2, inv_temp, out);
    else
        pp::k_response_logprobs<float><<<grid, pp::LP_THREADS, 0, s>>>(static_cast<const float *>(logits), V,
                                                                       token_ids, meta_d, c2, inv_temp, out);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_attn_fwd(const void *q, const void *k, const void *v, const void *meta_d, int64_t T, int32_t hq,
                      int32_t hkv, int32_t d, float softmax_scale, pp_dtype dt, void *o, float *lse,
                      void *workspace, int64_t ws_bytes, void *stream) {
    pp_status st = check_heads(T, hq, hkv, d);
    if (st != PP_OK) return st;
    if (T == 0) return PP_OK;
    if (!q || !k || !v || !meta_d || !o || !lse) return fail(PP_ERR_INVALID_ARG, "NULL pointer");
    if (dt != PP_BF16 && dt != PP_FP32) return fail(PP_ERR_INVALID_ARG, "unknown dtype %d", int(dt));
    int64_t need = 0;
    pp_workspace_bytes(PP_PASS_FWD, T, hq, hkv, d, &need);
    if (ws_bytes < need || !workspace) return fail(PP_ERR_WORKSPACE, "forward workspace too small");
    if (!(softmax_scale >= 0.f) || std::isinf(softmax_scale)) return fail(PP_ERR_INVALID_ARG, "bad softmax_scale");
    const float scale = softmax_scale == 0.f ? 1.f / std::sqrt(float(d)) : softmax_scale;
    DeviceInfo *di;
    if ((st = device_info(&di)) != PP_OK) return st;
    cudaStream_t s = as_stream(stream);
    if (dt == PP_FP32) {
        const size_t smem = size_t(2) * pp::FWD_BN * d * sizeof(float);
        const int64_t work = (T / pp::FWD_BM + 1024) * hq;
        if (d == 64) {
            PP_CUDA(cudaFuncSetAttribute(pp::k_attn_fwd_simt<float, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem)));
            pp::k_attn_fwd_simt<float, 64><<<grid_for(di->sm_count, 2, work), 128, smem, s>>>(
                static_cast<const float *>(q), static_cast<const float *>(k), static_cast<const float *>(v), meta_d,
                static_cast<float *>(o), lse, hq, hkv, scale);
        } else {
            PP_CUDA(cudaFuncSetAttribute(pp::k_attn_fwd_simt<float, 128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
            pp::k_attn_fwd_simt<float, 128><<<grid_for(di->sm_count, 1, work), 128, smem, s>>>(
                static_cast<const float *>(q), static_cast<const float *>(k), static_cast<const float *>(v), meta_d,
                static_cast<float *>(o), lse, hq, hkv, scale);
        }
        PP_CUDA(cudaGetLastError());
        return PP_OK;
    }
    CUtensorMap mq, mk, mv;
    if ((st = make_map_3d(&mq, q, T, hq, d, pp::FWD_BM)) != PP_OK) return st;
    if ((st = make_map_3d(&mk, k, T, hkv, d, pp::FWD_BN)) != PP_OK) return st;
    if ((st = make_map_3d(&mv, v, T, hkv, d, pp::FWD_BN)) != PP_OK) return st;
    if (reinterpret_cast<uintptr_t>(o) % 16) return fail(PP_ERR_INVALID_ARG, "o must be 16-byte aligned");
    const float sl2 = scale * 1.4426950408889634f;
    const int grid = di->sm_count;
    if (d == 128) {
        const size_t smem = sizeof(pp::FwdSmem<128>) + 1024;
        PP_CUDA(cudaFuncSetAttribute(pp::k_attn_fwd_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
        pp::k_attn_fwd_tc<128><<<grid, pp::FWD_THREADS, smem, s>>>(mq, mk, mv, meta_d,
                                                                     static_cast<__nv_bfloat16 *>(o), lse, hq, hkv, sl2);
    } else {
        const size_t smem = sizeof(pp::FwdSmem<64>) + 1024;
        PP_CUDA(cudaFuncSetAttribute(pp::k_attn_fwd_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
        pp::k_attn_fwd_tc<64><<<grid, pp::FWD_THREADS, smem, s>>>(mq, mk, mv, meta_d,
                                                                   static_cast<__nv_bfloat16 *>(o), lse, hq, hkv, sl2);
    }
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                      const void *dout, const void *meta_d, int64_t T, int32_t hq, int32_t hkv, int32_t d,
                      float softmax_scale, void *dq, void *dk, void *dv, void *workspace, int64_t ws_bytes,
                      void *stream) {
    pp_status st = check_heads(T, hq, hkv, d);
    if (st != PP_OK) return st;
    if (T == 0) return PP_OK;
    if (!q || !k || !v || !o || !lse || !dout || !meta_d || !dq || !dk || !dv)
        return fail(PP_ERR_INVALID_ARG, "NULL pointer");
    int64_t need = 0;
    pp_workspace_bytes(PP_PASS_BWD, T, hq, hkv, d, &need);
    if (ws_bytes < need || !workspace) return fail(PP_ERR_WORKSPACE, "backward workspace %lld < %lld bytes",
                                                   (long long)ws_bytes, (long long)need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(PP_ERR_INVALID_ARG, "workspace not 256-aligned");
    if (!(softmax_scale >= 0.f) || std::isinf(softmax_scale)) return fail(PP_ERR_INVALID_ARG, "bad softmax_scale");
    const float scale = softmax_scale == 0.f ? 1.f / std::sqrt(float(d)) : softmax_scale;
    DeviceInfo *di;
    if ((st = device_info(&di)) != PP_OK) return st;
    return pp::launch_bwd(q, k, v, o, lse, dout, meta_d, T, hq, hkv, d, scale, dq, dk, dv, workspace, ws_bytes,
                          di->sm_count, as_stream(stream), make_map_3d, make_map_3d_box, fail);
}

pp_status pp_attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const float *lse,
                              const void *dout, const void *meta_d, int64_t T, int32_t hq, int32_t hkv, int32_t d,
                              float softmax_scale, void *dq, void *dk, void *dv, void *stream) {
    pp_status st = check_heads(T, hq, hkv, d);
    if (st != PP_OK) return st;
    int64_t need = 0;
    if ((st = pp_workspace_bytes(PP_PASS_BWD, T, hq, hkv, d, &need)) != PP_OK) return st;
    if (need > PP_NOALLOC_SCRATCH_BYTES)
        return fail(PP_ERR_WORKSPACE,
                    "pp_attn_bwd_noalloc: these sizes need %lld bytes of scratch but the built-in array holds %lld; "
                    "call pp_attn_bwd with a caller workspace instead",
                    (long long)need, (long long)PP_NOALLOC_SCRATCH_BYTES);
    if (T == 0) return PP_OK;
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != PP_OK) return st;
    return pp_attn_bwd(q, k, v, o, lse, dout, meta_d, T, hq, hkv, d, softmax_scale, dq, dk, dv, scratch,
                       PP_NOALLOC_SCRATCH_BYTES, stream);
}

pp_status pp_selftest_bounded_wait(int64_t limit_ns, unsigned long long *waited_ns_d, void *stream) {
    if (limit_ns < 1000 || limit_ns > 2000000000ll)
        return fail(PP_ERR_INVALID_ARG, "limit_ns must be in [1e3, 2e9] (got %lld)", (long long)limit_ns);
    if (!waited_ns_d) return fail(PP_ERR_INVALID_ARG, "waited_ns_d is NULL");
    DeviceInfo *di;
    pp_status st = device_info(&di);
    if (st != PP_OK) return st;
    pp::k_selftest_wait<<<1, 32, 0, as_stream(stream)>>>(uint64_t(limit_ns), waited_ns_d);
    PP_CUDA(cudaGetLastError());
    return PP_OK;
}

pp_status pp_get_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize(as_stream(stream));
    if (e != cudaSuccess) return fail(PP_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
    int32_t word = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&word, pp::g_dev_err, sizeof(word));
    if (e != cudaSuccess) return fail(PP_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
    if (word == 0) return PP_OK;
    e = cudaMemcpyToSymbol(pp::g_dev_err, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(PP_ERR_CUDA, "clearing the device error word: %s", cudaGetErrorString(e));
    if (word & pp::DEVERR_TIMEOUT) return fail(PP_ERR_DEVICE_TIMEOUT, "a kernel's bounded wait ran out (0x%x)", word);
    return fail(PP_ERR_DEVICE_INPUT, "inconsistent descriptors, segment boundaries or token ids (0x%x)", word);
}

}  // extern "C"
