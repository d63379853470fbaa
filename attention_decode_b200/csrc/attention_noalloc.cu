// Decode attention for callers that cannot allocate device memory.
//
// nsnq_attn_decode needs a caller-provided workspace for the per-split
// softmax partials. Some callers have no way to obtain one: a plugin hosted
// by an engine that owns all device memory through its own allocator, a
// real-time loop where cudaMalloc (which may synchronise the device) is not
// allowed, or a plain C caller with no allocator at all. For them this file
// keeps the partials in a fixed array in device global memory instead.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds its kStaticScratchBytes until the process exits. In host
// code its name only stands in for the symbol, so the device address is
// looked up with cudaGetSymbolAddress with the device current: on every call
// whose stream is not capturing (the first call on a device must be one).
#include <mutex>

#include "../../include/nsnq.h"
#include "internal.h"

namespace {

// 4 MiB of fp32 partials: B * Hq * nsplit * 132 floats must fit, e.g. 16
// sequences x 32 heads x 5 context splits (1.35 MB) or 64 x 64 x 1 (2.2 MB).
constexpr size_t kStaticScratchBytes = size_t(4) << 20;

static __device__ __align__(256) unsigned char g_attn_partials[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_device_ptr[kMaxDevices] = {};

// Device address of g_attn_partials on the current device. A call whose
// stream is not capturing looks it up again every time (cheap once the module
// is loaded), so the address stays right after cudaDeviceReset, which can
// load the module elsewhere; a capturing call reuses the last address found
// on this device and sets *need_setup when there is none yet.
cudaError_t partials_on_current_device(cudaStream_t stream, void** out, bool* need_setup) {
    *need_setup = false;
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(stream, &cs);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (cs == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attn_partials);
        if (e != cudaSuccess) return e;
        g_device_ptr[dev] = p;
    } else if (g_device_ptr[dev] == nullptr) {
        *need_setup = true;
        return cudaSuccess;
    }
    *out = g_device_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" nsnq_status nsnq_attn_decode_noalloc(const void* q, nsnq_dtype q_dtype,
                                                nsnq_cache k_cache, nsnq_cache v_cache,
                                                nsnq_codebook k_cb, nsnq_codebook v_cb,
                                                const int32_t* seq_lens, int64_t max_len, int B,
                                                int Hq, int Hkv, int D, float softmax_scale,
                                                void* out, nsnq_dtype out_dtype,
                                                nsnq_stream stream) {
    // Shapes the regular entry point rejects are left to its own checks below.
    const size_t need = nsnq_attn_workspace(B, Hq, Hkv, D, max_len);
    if (need > kStaticScratchBytes) {
        return nsnq::set_error(NSNQ_ERR_WORKSPACE,
                               "nsnq_attn_decode_noalloc: this shape needs %zu bytes of split "
                               "partials but the fixed device array holds %zu; use "
                               "nsnq_attn_decode with a workspace, or fewer sequences, heads "
                               "or context",
                               need, kStaticScratchBytes);
    }
    void* partials = nullptr;
    bool need_setup = false;
    const cudaError_t e =
        partials_on_current_device(reinterpret_cast<cudaStream_t>(stream), &partials, &need_setup);
    if (e != cudaSuccess) {
        return nsnq::set_error(NSNQ_ERR_CUDA, "nsnq_attn_decode_noalloc setup: %s",
                               cudaGetErrorString(e));
    }
    if (need_setup) {
        return nsnq::set_error(NSNQ_ERR_INVALID_ARG,
                               "nsnq_attn_decode_noalloc: the stream is capturing and this "
                               "device has no array address yet; make one call on this device "
                               "before capturing");
    }
    // Every split writes all of its partial rows (empty splits write neutral
    // ones) before the combine reads them, so nothing needs clearing.
    return nsnq_attn_decode(q, q_dtype, k_cache, v_cache, k_cb, v_cb, seq_lens, max_len, B, Hq,
                            Hkv, D, softmax_scale, out, out_dtype, partials, kStaticScratchBytes,
                            stream);
}
