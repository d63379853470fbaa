// Host-side interfaces between the C ABI layer and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/nsnq.h"

namespace nsnq {

constexpr int kHeadDim = 128;      // the only head_dim the kernels support
constexpr int kNCentroids = 256;   // one byte per code
constexpr size_t kWsAlign = 256;
constexpr size_t kEncodeStatsBytes = 64;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Record a printf-style message as the calling thread's nsnq_last_error().
nsnq_status set_error(nsnq_status s, const char* fmt, ...);

// ---------------------------------------------------- launch set-up cache --
// Multiprocessor count of the current device, queried once per device.
int device_sm_count();

// The dynamic shared-memory limit of one kernel, set once per device (one
// bit per device in `ready`). A device reset drops the attribute; a launch
// that then fails with cudaErrorInvalidValue is retried once by launch_smem.
template <typename K>
cudaError_t ensure_smem(K kern, int bytes, std::atomic<unsigned long long>& ready, bool force) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? 1ull << dev : 0ull;
    if (!force && bit && (ready.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) ready.fetch_or(bit, std::memory_order_relaxed);
    return e;
}

// Launch kern<<<grid, block, smem, s>>>(args...) with its shared-memory limit
// set (once per device).
template <typename... P, typename... A>
cudaError_t launch_smem(void (*kern)(P...), std::atomic<unsigned long long>& ready, dim3 grid,
                        dim3 block, size_t smem, cudaStream_t s, A&&... args) {
    cudaError_t e = ensure_smem(kern, (int)smem, ready, false);
    if (e != cudaSuccess) return e;
    kern<<<grid, block, smem, s>>>(args...);
    e = cudaGetLastError();
    if (e == cudaErrorInvalidValue) {  // attribute lost (device reset): set it again, once
        e = ensure_smem(kern, (int)smem, ready, true);
        if (e != cudaSuccess) return e;
        kern<<<grid, block, smem, s>>>(args...);
        e = cudaGetLastError();
    }
    return e;
}

// launch_smem as a programmatic dependent launch: the kernel may start while
// the previous kernel in the stream finishes, and must execute
// griddepcontrol.wait before it reads what that kernel wrote.
template <typename... P, typename... A>
cudaError_t launch_smem_pdl(void (*kern)(P...), std::atomic<unsigned long long>& ready, dim3 grid,
                            dim3 block, size_t smem, cudaStream_t s, A&&... args) {
    cudaError_t e = ensure_smem(kern, (int)smem, ready, false);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e == cudaErrorInvalidValue) {  // attribute lost (device reset): set it again, once
        e = ensure_smem(kern, (int)smem, ready, true);
        if (e != cudaSuccess) return e;
        e = cudaLaunchKernelEx(&cfg, kern, args...);
    }
    return e;
}

// ------------------------------------------------ division by an invariant --
// n / d for 32-bit n and a divisor d >= 1 fixed per launch, as a multiply-high,
// a subtract, an add and two shifts (T. Granlund and P. Montgomery, "Division
// by Invariant Integers using Multiplication", PLDI 1994, section 4): with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1,
// q = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0), t = mulhi(m, n), exact
// for every 32-bit n.
struct FastDiv {
    uint32_t d, m, s1, s2;
};
inline FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < d) ++l;
    const uint64_t m = (((1ull << 32) * ((1ull << l) - d)) / d) + 1;
    return {d, (uint32_t)m, l < 1 ? l : 1u, l > 0 ? l - 1 : 0u};
}
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
    const uint32_t t = __umulhi(n, f.m);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}
#endif

// ------------------------------------------------------------------ encode --
struct EncodeArgs {
    const void* x;
    int x_bf16;
    int B, H;
    int64_t T;
    int64_t sb, sh, st;
    int64_t t_offset;
    int given_shift;
    int adaptive;  // scale adjustment folded into s2
    int dq;        // double quantization of s1 and o
    float* s1_grid;  // [B][H][2] (lo, step) of the log2 s1 grid
    const float* C;
    int sub;
    const void* index;  // search index (sub == 4, walk search)
    int tc_search;      // sub == 4: score every codeword on the tensor cores (no index)
    uint8_t* codes;
    float* scales;
    float* shift;
    int64_t cap;
    uint32_t* s1_levels;  // packed double-quantized form: 4-bit s1 levels, scales = s2 only
    // workspace views
    unsigned long long* stats;  // [8]
    double* partial;            // [B][H][nchunk1][128]
    double* o64;                // [B][H][128]
    double* minmax;             // [B][H][nchunk1][2] least / largest log2 s1 per chunk
    unsigned* head_done;        // [B][H] chunks of pass 1 finished (zeroed per call)
    int zero_stats;             // the pass-2 kernel zeroes stats (no memset before the call)
    int nchunk1;
    int64_t chunk1;
    // Two tensors in one call (keys and values, nsnq_encode_kv): batches
    // [0, B1) of the grid are the first tensor (x, codes, ...), [B1, B) the
    // second (x2, codes2, ...), B = 2 B1. The workspace is indexed by the
    // grid's (b, h); the caches by the tensor's own. One tensor: B1 = B.
    int B1;
    const void* x2;
    uint8_t* codes2;
    float* scales2;
    float* shift2;
    uint32_t* s1_levels2;
    float* s1_grid2;
    // Set by the pass-2 launchers: the divisions of the work decomposition
    // (work items per head, heads per batch); every index is below 2^31.
    FastDiv div_items;
    FastDiv div_H;
};

#ifdef __CUDACC__
// Grid head bh = b * H + h (b < B) belongs to the second tensor when
// b >= B1; its cache row block is then bh - B1 * H.
__device__ __forceinline__ bool enc_second(const EncodeArgs& a, int64_t bh) {
    return bh >= (int64_t)a.B1 * a.H;
}
__device__ __forceinline__ int64_t enc_cbh(const EncodeArgs& a, int64_t bh) {
    return enc_second(a, bh) ? bh - (int64_t)a.B1 * a.H : bh;
}
// First element of head (b, h) of the tensor that grid batch b belongs to.
template <typename XT>
__device__ __forceinline__ const XT* enc_head(const EncodeArgs& a, int b, int h) {
    const bool sec = b >= a.B1;
    return reinterpret_cast<const XT*>(sec ? a.x2 : a.x) + (int64_t)(sec ? b - a.B1 : b) * a.sb +
           (int64_t)h * a.sh;
}
// The cache arrays of the tensor selected by `sec`.
__device__ __forceinline__ uint8_t* enc_codes(const EncodeArgs& a, bool sec) {
    return sec ? a.codes2 : a.codes;
}
__device__ __forceinline__ float* enc_scales(const EncodeArgs& a, bool sec) {
    return sec ? a.scales2 : a.scales;
}
__device__ __forceinline__ float* enc_shift(const EncodeArgs& a, bool sec) {
    return sec ? a.shift2 : a.shift;
}
__device__ __forceinline__ uint32_t* enc_s1_levels(const EncodeArgs& a, bool sec) {
    return sec ? a.s1_levels2 : a.s1_levels;
}
__device__ __forceinline__ float* enc_s1_grid(const EncodeArgs& a, bool sec) {
    return sec ? a.s1_grid2 : a.s1_grid;
}
#endif

struct EncodePlan {
    int nchunk1;
    int64_t chunk1;
    size_t reset_bytes;  // leading workspace bytes zeroed before each call
    size_t partial_off, o64_off, minmax_off, total;
};

EncodePlan plan_encode(int B, int H, int64_t T);
cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s);
cudaError_t launch_encode_pruned(const EncodeArgs& a, cudaStream_t s);
// Pass 2 of calls with at most kSmallEncode token-heads: one warp per
// token-head, fp64 throughout (a decode step's appends).
constexpr int64_t kSmallEncode = 1024;
cudaError_t launch_encode_small(const EncodeArgs& a, cudaStream_t s);
// Pass 2 with every codeword scored on the tensor cores: sub == 8, or sub == 4
// with tc_search (encode1_tc.cu).
cudaError_t launch_encode_tc(const EncodeArgs& a, cudaStream_t s);
size_t index_bytes();
cudaError_t launch_index_build(const float* C, void* index, cudaStream_t s);
cudaError_t launch_codebook_q4(const float* in, float* out, uint8_t* levels, double* grid, int n,
                               cudaStream_t s);

// ----------------------------------------------------------------- dequant --
struct DequantArgs {
    const uint8_t* codes;
    const float* scales;
    const float* shift;
    int64_t cap;
    const uint32_t* s1_levels;  // packed form (scales = s2 only), or NULL
    const float* s1_grid;
    const float* C;
    int sub;
    int B, H;
    int64_t t0, T;
    float* out;
};
cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t s);

// --------------------------------------------------------------- attention --
constexpr int kPartStride = 132;  // 128 rotated-domain values + (m, l, beta, pad)

struct AttnPlan {
    int gc;          // query heads per CTA
    int ngroups;     // head groups per kv-head
    int64_t units;   // (batch, kv-head, head group) triples
    int64_t L;       // virtual tokens per unit (max_len)
    int ctas;        // CTAs of the split kernel (one per SM)
    int nslot;       // partial rows per (batch, query head)
    size_t total;
};

AttnPlan plan_attention(int B, int Hq, int Hkv, int64_t max_len);

struct AttnArgs {
    const void* q;
    int q_bf16;
    const uint8_t* kcodes;
    const float* kscales;
    const float* kshift;
    int64_t kcap;
    const float* kC;
    int ksub;
    const uint32_t* klevels;  // packed double-quantized K cache (scales = s2 only), or NULL
    const float* kgrid;
    const uint8_t* vcodes;
    const float* vscales;
    const float* vshift;
    int64_t vcap;
    const float* vC;
    int vsub;
    const uint32_t* vlevels;  // packed double-quantized V cache, or NULL
    const float* vgrid;
    const int32_t* seq_lens;
    int64_t max_len;
    int B, Hq, Hkv;
    float scale_log2;
    void* out;
    int out_bf16;
    float* part;
    AttnPlan plan;
    // full-precision residual window ([B][Hkv][rcap][D]; rcap = 0: none)
    const void* rk;
    const void* rv;
    int r_bf16;
    const int32_t* res_lens;
    int64_t rcap;
    // keys quantized before RoPE: rotary base (the split kernel of attention_rope.cu)
    double rope_base;
};
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_attn_combine(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_attention_rope(const AttnArgs& a, cudaStream_t s);

struct ResWriteArgs {
    const void* x;
    int x_bf16;
    int B, H;
    int64_t T;
    int64_t sb, sh, st;
    int64_t t_offset;
    void* buf;
    int buf_bf16;
    int64_t cap;
};
cudaError_t launch_residual_write(const ResWriteArgs& a, cudaStream_t s);

}  // namespace nsnq
