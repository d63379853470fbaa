// C ABI of the NSNQuant library: argument validation, workspace planning and
// kernel launches. Every check runs on the host before anything is launched.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include "../../include/nsnq.h"
#include "internal.h"
#include "vq_index.cuh"

namespace {

thread_local char g_err[512] = "";

nsnq_status fail(nsnq_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

nsnq_status ok() {
    g_err[0] = '\0';
    return NSNQ_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

nsnq_status cuda_fail(cudaError_t e, const char* what) {
    return fail(NSNQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

nsnq_status check_codebook(const nsnq_codebook& cb, const char* name) {
    if (!cb.centroids) return fail(NSNQ_ERR_INVALID_ARG, "%s.centroids is NULL", name);
    if (!aligned(cb.centroids, 16))
        return fail(NSNQ_ERR_INVALID_ARG, "%s.centroids must be 16-byte aligned", name);
    if (cb.n_centroids != nsnq::kNCentroids)
        return fail(NSNQ_ERR_UNSUPPORTED, "%s.n_centroids = %d (only 256 is supported)", name,
                    cb.n_centroids);
    if (cb.sub_dim != 4 && cb.sub_dim != 8)
        return fail(NSNQ_ERR_UNSUPPORTED, "%s.sub_dim = %d (4 or 8 supported)", name, cb.sub_dim);
    return NSNQ_OK;
}

nsnq_status check_cache(const nsnq_cache& c, const char* name, bool need_shift) {
    if (!c.codes || !c.scales || (need_shift && !c.shift))
        return fail(NSNQ_ERR_INVALID_ARG, "%s has a NULL buffer", name);
    if (!aligned(c.codes, 16) || !aligned(c.scales, 16) || (c.shift && !aligned(c.shift, 16)))
        return fail(NSNQ_ERR_INVALID_ARG, "%s buffers must be 16-byte aligned", name);
    if (c.cap < 0) return fail(NSNQ_ERR_INVALID_ARG, "%s.cap = %lld < 0", name, (long long)c.cap);
    if (c.s1_levels && (!c.s1_grid || !aligned(c.s1_levels, 4) || !aligned(c.s1_grid, 8)))
        return fail(NSNQ_ERR_INVALID_ARG,
                    "%s: a packed cache (s1_levels) needs s1_grid; s1_levels 4-byte and s1_grid "
                    "8-byte aligned", name);
    return NSNQ_OK;
}

}  // namespace

namespace nsnq {
int device_sm_count() {
    static std::atomic<int> cached[64] = {};
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return 148;
    }
    if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

nsnq_status set_error(nsnq_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}
}  // namespace nsnq

extern "C" {

const char* nsnq_status_string(nsnq_status s) {
    switch (s) {
        case NSNQ_OK: return "NSNQ_OK";
        case NSNQ_ERR_INVALID_ARG: return "NSNQ_ERR_INVALID_ARG";
        case NSNQ_ERR_UNSUPPORTED: return "NSNQ_ERR_UNSUPPORTED";
        case NSNQ_ERR_WORKSPACE: return "NSNQ_ERR_WORKSPACE";
        case NSNQ_ERR_CUDA: return "NSNQ_ERR_CUDA";
    }
    return "NSNQ_ERR_UNKNOWN";
}

const char* nsnq_last_error(void) { return g_err; }

size_t nsnq_codebook_index_bytes(int sub_dim) {
    return sub_dim == 4 ? nsnq::index_bytes() : 0;
}

nsnq_status nsnq_codebook_index_build(nsnq_codebook cb, void* index, size_t index_bytes,
                                      nsnq_stream stream) {
    nsnq_status s = check_codebook(cb, "cb");
    if (s != NSNQ_OK) return s;
    if (cb.sub_dim != 4) return fail(NSNQ_ERR_UNSUPPORTED, "only sub_dim 4 codebooks take an index");
    if (!index || !aligned(index, 16))
        return fail(NSNQ_ERR_INVALID_ARG, "index NULL or not 16-byte aligned");
    if (index_bytes < nsnq::index_bytes())
        return fail(NSNQ_ERR_WORKSPACE, "index of %zu bytes needed, %zu given", nsnq::index_bytes(),
                    index_bytes);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = nsnq::launch_index_build(cb.centroids, index, st);
    if (e != cudaSuccess) return cuda_fail(e, "index build launch");
    uint32_t hdr[4] = {0, 0, 0, 0};
    e = cudaMemcpyAsync(hdr, index, sizeof(hdr), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "index build");
    if (hdr[2] != 0)
        return fail(NSNQ_ERR_UNSUPPORTED, "codebook index needs %u list entry pairs (limit %d)", hdr[1],
                    nsnq::kMaxPairs);
    return ok();
}

nsnq_status nsnq_codebook_quantize4(const float* centroids, float* out, uint8_t* levels,
                                    double* grid, int n_centroids, int sub_dim,
                                    nsnq_stream stream) {
    if (n_centroids != nsnq::kNCentroids)
        return fail(NSNQ_ERR_UNSUPPORTED, "n_centroids = %d (only 256 is supported)", n_centroids);
    if (sub_dim != 4 && sub_dim != 8)
        return fail(NSNQ_ERR_UNSUPPORTED, "sub_dim = %d (4 or 8 supported)", sub_dim);
    if (!centroids || !out) return fail(NSNQ_ERR_INVALID_ARG, "centroids or out is NULL");
    if (!aligned(centroids, 4) || !aligned(out, 4) || (grid && !aligned(grid, 8)))
        return fail(NSNQ_ERR_INVALID_ARG, "centroids/out must be 4-byte and grid 8-byte aligned");
    cudaError_t e = nsnq::launch_codebook_q4(centroids, out, levels, grid, n_centroids * sub_dim,
                                             reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "codebook quantize4 launch");
    return ok();
}

size_t nsnq_encode_workspace(int B, int H, int64_t T, int D) {
    if (B < 0 || H < 0 || T < 0 || D != nsnq::kHeadDim) return 0;
    return nsnq::plan_encode(B, H, T).total;
}

namespace {

// Checks of one tensor's cache for an encode call (shared by both entry points).
nsnq_status check_encode_cache(const nsnq_cache& cache, const char* name, bool dq, int64_t T,
                               int64_t t_offset) {
    if (dq && (!cache.s1_grid || !aligned(cache.s1_grid, 8)))
        return fail(NSNQ_ERR_INVALID_ARG, "double quantization needs %s.s1_grid (8-byte aligned)", name);
    if (cache.s1_levels && !dq)
        return fail(NSNQ_ERR_INVALID_ARG,
                    "a packed cache (%s.s1_levels) holds double-quantized s1 only: pass "
                    "NSNQ_ENCODE_DOUBLE_QUANT", name);
    nsnq_status s = check_cache(cache, name, true);
    if (s != NSNQ_OK) return s;
    if (t_offset < 0 || t_offset > cache.cap || T > cache.cap - t_offset)
        return fail(NSNQ_ERR_INVALID_ARG, "positions [%lld, %lld) exceed %s capacity %lld",
                    (long long)t_offset, (long long)(t_offset + T), name, (long long)cache.cap);
    return NSNQ_OK;
}

// One tensor (x2 == NULL) or two of one shape sharing every launch: the
// second tensor's heads follow the first's as batches [B, 2B) of the grid.
nsnq_status encode_impl(const void* x, const void* x2, nsnq_dtype x_dtype, int B, int H, int64_t T,
                        int D, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                        int64_t t_offset, nsnq_shift_mode mode, unsigned flags, nsnq_codebook cb,
                        const nsnq_cache& cache, const nsnq_cache* cache2, void* workspace,
                        size_t workspace_bytes, nsnq_stream stream) {
    const bool pair = cache2 != nullptr;
    if (D != nsnq::kHeadDim) return fail(NSNQ_ERR_UNSUPPORTED, "D = %d (only 128 is supported)", D);
    if (x_dtype != NSNQ_F32 && x_dtype != NSNQ_BF16)
        return fail(NSNQ_ERR_UNSUPPORTED, "x_dtype = %d", (int)x_dtype);
    if (mode != NSNQ_SHIFT_COMPUTE && mode != NSNQ_SHIFT_GIVEN)
        return fail(NSNQ_ERR_INVALID_ARG, "shift mode = %d", (int)mode);
    if (flags & ~(unsigned)(NSNQ_ENCODE_ADAPTIVE_SCALE | NSNQ_ENCODE_DOUBLE_QUANT | NSNQ_ENCODE_TC_SEARCH))
        return fail(NSNQ_ERR_INVALID_ARG, "unknown encode flags 0x%x", flags);
    const bool dq = (flags & NSNQ_ENCODE_DOUBLE_QUANT) != 0;
    if (B < 0 || H < 0 || T < 0)
        return fail(NSNQ_ERR_INVALID_ARG, "negative size B=%d H=%d T=%lld", B, H, (long long)T);
    if (B > (pair ? 32767 : 65535) || H > 65535)
        return fail(NSNQ_ERR_UNSUPPORTED, "B or H above %s", pair ? "32767 / 65535" : "65535");
    nsnq_status s = check_codebook(cb, "cb");
    if (s != NSNQ_OK) return s;
    const bool tc_search = (flags & NSNQ_ENCODE_TC_SEARCH) != 0;
    if (cb.sub_dim == 4 && !tc_search && (!cb.index || !aligned(cb.index, 16)))
        return fail(NSNQ_ERR_INVALID_ARG,
                    "cb.index is NULL or misaligned: build it with nsnq_codebook_index_build "
                    "(or pass NSNQ_ENCODE_TC_SEARCH)");
    s = check_encode_cache(cache, pair ? "cache_k" : "cache", dq, T, t_offset);
    if (s != NSNQ_OK) return s;
    if (pair) {
        s = check_encode_cache(*cache2, "cache_v", dq, T, t_offset);
        if (s != NSNQ_OK) return s;
        if (cache2->cap != cache.cap)
            return fail(NSNQ_ERR_INVALID_ARG, "cache_k.cap = %lld and cache_v.cap = %lld differ",
                        (long long)cache.cap, (long long)cache2->cap);
        if ((cache2->s1_levels != nullptr) != (cache.s1_levels != nullptr))
            return fail(NSNQ_ERR_INVALID_ARG, "cache_k and cache_v must both be packed or both not");
        if (cache2->codes == cache.codes || cache2->scales == cache.scales || cache2->shift == cache.shift ||
            (cache.s1_levels && cache2->s1_levels == cache.s1_levels) ||
            (cache.s1_grid && cache2->s1_grid == cache.s1_grid))
            return fail(NSNQ_ERR_INVALID_ARG, "cache_k and cache_v share a buffer");
    }
    if (B == 0 || H == 0 || T == 0) return ok();
    if (!x || (pair && !x2)) return fail(NSNQ_ERR_INVALID_ARG, "%s is NULL", pair ? "x_k or x_v" : "x");
    const int64_t esz = x_dtype == NSNQ_BF16 ? 2 : 4;
    if (!aligned(x, 16) || (pair && !aligned(x2, 16)) || (stride_b * esz) % 16 || (stride_h * esz) % 16 ||
        (stride_t * esz) % 16)
        return fail(NSNQ_ERR_INVALID_ARG, "x and its strides must be 16-byte aligned");
    if (stride_b < 0 || stride_h < 0 || stride_t < D)
        return fail(NSNQ_ERR_INVALID_ARG, "strides must be non-negative with stride_t >= D");
    const int Bg = pair ? 2 * B : B;  // batches of the grid
    // work indices are 32-bit (2^31 token-heads of bf16 input are 550 GB)
    if ((int64_t)Bg * H * T >= (int64_t)1 << 31)
        return fail(NSNQ_ERR_UNSUPPORTED, "%lld token-heads in one call (limit 2^31)",
                    (long long)Bg * H * T);
    const nsnq::EncodePlan plan = nsnq::plan_encode(Bg, H, T);
    if (!workspace || workspace_bytes < plan.total)
        return fail(NSNQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", plan.total,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, nsnq::kWsAlign))
        return fail(NSNQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");

    nsnq::EncodeArgs a{};
    a.x = x;
    a.x_bf16 = x_dtype == NSNQ_BF16;
    a.B = Bg; a.H = H; a.T = T;
    a.sb = stride_b; a.sh = stride_h; a.st = stride_t;
    a.t_offset = t_offset;
    a.given_shift = mode == NSNQ_SHIFT_GIVEN;
    a.adaptive = (flags & NSNQ_ENCODE_ADAPTIVE_SCALE) ? 1 : 0;
    a.dq = dq ? 1 : 0;
    a.s1_grid = cache.s1_grid;
    a.C = cb.centroids;
    a.sub = cb.sub_dim;
    a.index = cb.index;
    a.tc_search = tc_search ? 1 : 0;
    a.codes = cache.codes; a.scales = cache.scales; a.shift = cache.shift; a.cap = cache.cap;
    a.s1_levels = cache.s1_levels;
    a.B1 = B;
    const nsnq_cache& c2 = pair ? *cache2 : cache;
    a.x2 = pair ? x2 : x;
    a.codes2 = c2.codes; a.scales2 = c2.scales; a.shift2 = c2.shift;
    a.s1_levels2 = c2.s1_levels; a.s1_grid2 = c2.s1_grid;
    char* ws = static_cast<char*>(workspace);
    a.stats = reinterpret_cast<unsigned long long*>(ws);
    a.partial = reinterpret_cast<double*>(ws + plan.partial_off);
    a.o64 = reinterpret_cast<double*>(ws + plan.o64_off);
    a.minmax = reinterpret_cast<double*>(ws + plan.minmax_off);
    a.head_done = reinterpret_cast<unsigned*>(ws + nsnq::kEncodeStatsBytes);
    a.nchunk1 = plan.nchunk1;
    a.chunk1 = plan.chunk1;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // A small shift-given call (a decode step's appends) uses no counter: its
    // kernel zeroes the stats block itself, which saves the memset.
    a.zero_stats = a.given_shift && (int64_t)Bg * H * T <= nsnq::kSmallEncode;
    cudaError_t e = a.zero_stats ? cudaSuccess : cudaMemsetAsync(ws, 0, plan.reset_bytes, st);
    if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
    e = nsnq::launch_encode(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "encode launch");
    return ok();
}

}  // namespace

nsnq_status nsnq_encode(const void* x, nsnq_dtype x_dtype, int B, int H, int64_t T, int D,
                        int64_t stride_b, int64_t stride_h, int64_t stride_t, int64_t t_offset,
                        nsnq_shift_mode mode, unsigned flags, nsnq_codebook cb, nsnq_cache cache,
                        void* workspace, size_t workspace_bytes, nsnq_stream stream) {
    return encode_impl(x, nullptr, x_dtype, B, H, T, D, stride_b, stride_h, stride_t, t_offset, mode,
                       flags, cb, cache, nullptr, workspace, workspace_bytes, stream);
}

size_t nsnq_encode_kv_workspace(int B, int H, int64_t T, int D) {
    if (B < 0 || B > 32767 || H < 0 || T < 0 || D != nsnq::kHeadDim) return 0;
    return nsnq::plan_encode(2 * B, H, T).total;
}

nsnq_status nsnq_encode_kv(const void* x_k, const void* x_v, nsnq_dtype x_dtype, int B, int H,
                           int64_t T, int D, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                           int64_t t_offset, nsnq_shift_mode mode, unsigned flags, nsnq_codebook cb,
                           nsnq_cache cache_k, nsnq_cache cache_v, void* workspace,
                           size_t workspace_bytes, nsnq_stream stream) {
    return encode_impl(x_k, x_v, x_dtype, B, H, T, D, stride_b, stride_h, stride_t, t_offset, mode,
                       flags, cb, cache_k, &cache_v, workspace, workspace_bytes, stream);
}

nsnq_status nsnq_dequant(nsnq_cache cache, nsnq_codebook cb, int B, int H, int64_t t0, int64_t T,
                         int D, float* out, nsnq_stream stream) {
    if (D != nsnq::kHeadDim) return fail(NSNQ_ERR_UNSUPPORTED, "D = %d (only 128 is supported)", D);
    if (B < 0 || H < 0 || T < 0 || t0 < 0)
        return fail(NSNQ_ERR_INVALID_ARG, "negative size or offset");
    nsnq_status s = check_codebook(cb, "cb");
    if (s != NSNQ_OK) return s;
    s = check_cache(cache, "cache", true);
    if (s != NSNQ_OK) return s;
    if (t0 > cache.cap || T > cache.cap - t0)
        return fail(NSNQ_ERR_INVALID_ARG, "positions [%lld, %lld) exceed cache capacity %lld",
                    (long long)t0, (long long)(t0 + T), (long long)cache.cap);
    if (B == 0 || H == 0 || T == 0) return ok();
    if (!out || !aligned(out, 16)) return fail(NSNQ_ERR_INVALID_ARG, "out NULL or not 16-byte aligned");
    nsnq::DequantArgs a{};
    a.codes = cache.codes; a.scales = cache.scales; a.shift = cache.shift; a.cap = cache.cap;
    a.s1_levels = cache.s1_levels; a.s1_grid = cache.s1_grid;
    a.C = cb.centroids; a.sub = cb.sub_dim;
    a.B = B; a.H = H; a.t0 = t0; a.T = T;
    a.out = out;
    cudaError_t e = nsnq::launch_dequant(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
    return ok();
}

size_t nsnq_attn_workspace(int B, int Hq, int Hkv, int D, int64_t max_len) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D != nsnq::kHeadDim || max_len < 0) return 0;
    return nsnq::plan_attention(B, Hq, Hkv, max_len).total;
}

// Validates a decode-attention call and fills its arguments; *empty is set
// when there is nothing to launch (B = 0).
static nsnq_status attn_args(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                             nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                             const int32_t* seq_lens, int64_t max_len, nsnq_residual res,
                             int B, int Hq, int Hkv, int D, float softmax_scale, void* out,
                             nsnq_dtype out_dtype, void* workspace, size_t workspace_bytes,
                             nsnq::AttnArgs& a, bool* empty) {
    *empty = false;
    if (D != nsnq::kHeadDim) return fail(NSNQ_ERR_UNSUPPORTED, "D = %d (only 128 is supported)", D);
    if ((q_dtype != NSNQ_F32 && q_dtype != NSNQ_BF16) ||
        (out_dtype != NSNQ_F32 && out_dtype != NSNQ_BF16))
        return fail(NSNQ_ERR_UNSUPPORTED, "q/out dtype must be NSNQ_F32 or NSNQ_BF16");
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv)
        return fail(NSNQ_ERR_INVALID_ARG, "need B >= 0 and Hq a positive multiple of Hkv (B=%d Hq=%d Hkv=%d)",
                    B, Hq, Hkv);
    if (B > 65535 || Hq > 65535) return fail(NSNQ_ERR_UNSUPPORTED, "B or Hq above 65535");
    if (!isfinite(softmax_scale)) return fail(NSNQ_ERR_INVALID_ARG, "softmax_scale is not finite");
    nsnq_status s = check_codebook(k_cb, "k_cb");
    if (s != NSNQ_OK) return s;
    s = check_codebook(v_cb, "v_cb");
    if (s != NSNQ_OK) return s;
    s = check_cache(k_cache, "k_cache", true);
    if (s != NSNQ_OK) return s;
    s = check_cache(v_cache, "v_cache", true);
    if (s != NSNQ_OK) return s;
    if (max_len < 0 || max_len > k_cache.cap || max_len > v_cache.cap)
        return fail(NSNQ_ERR_INVALID_ARG, "max_len = %lld must be in [0, min(cap)]",
                    (long long)max_len);
    if (res.cap < 0) return fail(NSNQ_ERR_INVALID_ARG, "res.cap = %lld < 0", (long long)res.cap);
    if (res.cap > 0) {
        if (res.dtype != NSNQ_F32 && res.dtype != NSNQ_BF16)
            return fail(NSNQ_ERR_UNSUPPORTED, "res.dtype must be NSNQ_F32 or NSNQ_BF16");
        if (B > 0 && (!res.k || !res.v || !res.lens))
            return fail(NSNQ_ERR_INVALID_ARG, "res.k, res.v or res.lens is NULL");
        if (!aligned(res.k, 16) || !aligned(res.v, 16) || !aligned(res.lens, 4))
            return fail(NSNQ_ERR_INVALID_ARG, "res.k and res.v must be 16-byte aligned");
    }
    if (B == 0) {
        *empty = true;
        return ok();
    }
    if (!q || !out || !seq_lens) return fail(NSNQ_ERR_INVALID_ARG, "q, out or seq_lens is NULL");
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(seq_lens, 4))
        return fail(NSNQ_ERR_INVALID_ARG, "q and out must be 16-byte aligned");
    const nsnq::AttnPlan plan = nsnq::plan_attention(B, Hq, Hkv, max_len);
    if (!workspace || workspace_bytes < plan.total)
        return fail(NSNQ_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", plan.total,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned(workspace, nsnq::kWsAlign))
        return fail(NSNQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    a = nsnq::AttnArgs{};
    a.q = q; a.q_bf16 = q_dtype == NSNQ_BF16;
    a.kcodes = k_cache.codes; a.kscales = k_cache.scales; a.kshift = k_cache.shift;
    a.kcap = k_cache.cap; a.kC = k_cb.centroids; a.ksub = k_cb.sub_dim;
    a.klevels = k_cache.s1_levels; a.kgrid = k_cache.s1_grid;
    a.vcodes = v_cache.codes; a.vscales = v_cache.scales; a.vshift = v_cache.shift;
    a.vcap = v_cache.cap; a.vC = v_cb.centroids; a.vsub = v_cb.sub_dim;
    a.vlevels = v_cache.s1_levels; a.vgrid = v_cache.s1_grid;
    a.seq_lens = seq_lens; a.max_len = max_len;
    a.B = B; a.Hq = Hq; a.Hkv = Hkv;
    const float scale = softmax_scale == 0.f ? 1.0f / sqrtf((float)D) : softmax_scale;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.out = out; a.out_bf16 = out_dtype == NSNQ_BF16;
    a.part = static_cast<float*>(workspace);
    a.plan = plan;
    if (res.cap > 0) {
        a.rk = res.k; a.rv = res.v; a.r_bf16 = res.dtype == NSNQ_BF16;
        a.res_lens = res.lens; a.rcap = res.cap;
    }
    return NSNQ_OK;
}

nsnq_status nsnq_attn_decode_res(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                                 nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                                 const int32_t* seq_lens, int64_t max_len, nsnq_residual res,
                                 int B, int Hq, int Hkv, int D, float softmax_scale, void* out,
                                 nsnq_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                 nsnq_stream stream) {
    nsnq::AttnArgs a;
    bool empty = false;
    const nsnq_status s = attn_args(q, q_dtype, k_cache, v_cache, k_cb, v_cb, seq_lens, max_len, res, B,
                                    Hq, Hkv, D, softmax_scale, out, out_dtype, workspace,
                                    workspace_bytes, a, &empty);
    if (s != NSNQ_OK || empty) return s;
    cudaError_t e = nsnq::launch_attention(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return ok();
}

nsnq_status nsnq_attn_decode_rope(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                                  nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                                  const int32_t* seq_lens, int64_t max_len, double rope_base,
                                  int B, int Hq, int Hkv, int D, float softmax_scale, void* out,
                                  nsnq_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                  nsnq_stream stream) {
    if (!isfinite(rope_base) || !(rope_base > 1.0))
        return fail(NSNQ_ERR_INVALID_ARG, "rope_base = %g must be finite and > 1", rope_base);
    nsnq::AttnArgs a;
    bool empty = false;
    nsnq_residual none{};
    const nsnq_status s = attn_args(q, q_dtype, k_cache, v_cache, k_cb, v_cb, seq_lens, max_len, none,
                                    B, Hq, Hkv, D, softmax_scale, out, out_dtype, workspace,
                                    workspace_bytes, a, &empty);
    if (s != NSNQ_OK || empty) return s;
    a.rope_base = rope_base;
    cudaError_t e = nsnq::launch_attention_rope(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "attention (rope) launch");
    return ok();
}

nsnq_status nsnq_attn_decode(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                             nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                             const int32_t* seq_lens, int64_t max_len, int B, int Hq, int Hkv,
                             int D, float softmax_scale, void* out, nsnq_dtype out_dtype,
                             void* workspace, size_t workspace_bytes, nsnq_stream stream) {
    nsnq_residual none{};
    return nsnq_attn_decode_res(q, q_dtype, k_cache, v_cache, k_cb, v_cb, seq_lens, max_len, none,
                                B, Hq, Hkv, D, softmax_scale, out, out_dtype, workspace,
                                workspace_bytes, stream);
}

nsnq_status nsnq_residual_write(const void* x, nsnq_dtype x_dtype, int B, int H, int64_t T, int D,
                                int64_t stride_b, int64_t stride_h, int64_t stride_t,
                                int64_t t_offset, void* buf, nsnq_dtype buf_dtype, int64_t cap,
                                nsnq_stream stream) {
    if (D != nsnq::kHeadDim) return fail(NSNQ_ERR_UNSUPPORTED, "D = %d (only 128 is supported)", D);
    if ((x_dtype != NSNQ_F32 && x_dtype != NSNQ_BF16) ||
        (buf_dtype != NSNQ_F32 && buf_dtype != NSNQ_BF16))
        return fail(NSNQ_ERR_UNSUPPORTED, "x/buf dtype must be NSNQ_F32 or NSNQ_BF16");
    if (B < 0 || H < 0 || T < 0 || cap < 0)
        return fail(NSNQ_ERR_INVALID_ARG, "negative size B=%d H=%d T=%lld cap=%lld", B, H,
                    (long long)T, (long long)cap);
    if (t_offset < 0 || t_offset > cap || T > cap - t_offset)
        return fail(NSNQ_ERR_INVALID_ARG, "rows [%lld, %lld) exceed capacity %lld",
                    (long long)t_offset, (long long)(t_offset + T), (long long)cap);
    if (B == 0 || H == 0 || T == 0) return ok();
    if (!x || !buf) return fail(NSNQ_ERR_INVALID_ARG, "x or buf is NULL");
    const int64_t esz = x_dtype == NSNQ_BF16 ? 2 : 4;
    if (!aligned(x, 16) || (stride_b * esz) % 16 || (stride_h * esz) % 16 || (stride_t * esz) % 16)
        return fail(NSNQ_ERR_INVALID_ARG, "x and its strides must be 16-byte aligned");
    if (stride_b < 0 || stride_h < 0 || stride_t < D)
        return fail(NSNQ_ERR_INVALID_ARG, "strides must be non-negative with stride_t >= D");
    if (!aligned(buf, 16)) return fail(NSNQ_ERR_INVALID_ARG, "buf must be 16-byte aligned");
    nsnq::ResWriteArgs a{};
    a.x = x; a.x_bf16 = x_dtype == NSNQ_BF16;
    a.B = B; a.H = H; a.T = T;
    a.sb = stride_b; a.sh = stride_h; a.st = stride_t;
    a.t_offset = t_offset;
    a.buf = buf; a.buf_bf16 = buf_dtype == NSNQ_BF16; a.cap = cap;
    cudaError_t e = nsnq::launch_residual_write(a, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "residual write launch");
    return ok();
}

}  // extern "C"
