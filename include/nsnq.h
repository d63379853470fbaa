/*
 * nsnq.h -- C ABI of the B200 (sm_100a) NSNQuant KV-cache library.
 *
 * NSNQuant ("NSNQuant: A Double Normalization Approach for Calibration-Free
 * Low-Bit Vector Quantization of KV Cache", as summarised on gist.science,
 * Technical Summary) quantizes each key/value token in four steps:
 *   (Methodology §1) Normalize-Shift-Normalize: s1 = ||x||/sqrt(D), y = x/s1;
 *       o = channel-wise mean of y over the prompt; z = y - o;
 *       s2 = ||z||/sqrt(D), u = z/s2 (so ||u|| = sqrt(D));
 *   (Methodology §2) w = H u with the naive orthonormal Hadamard matrix H
 *       (Sylvester order, entries +-1/sqrt(D));
 *   (Methodology §3) each sub-vector w[j*g:(j+1)*g] is replaced by the index
 *       of its nearest codeword in one global 256-entry codebook built by
 *       k-means on standard-normal samples (g = 8: 1 bit/coordinate,
 *       g = 4: 2 bits/coordinate);
 *   (Methodology §4) attention scores and outputs are computed from the codes
 *       and the byproducts (s1, s2, o) directly.
 * Reconstruction: x_hat = s1 * (s2 * H w_hat + o).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers unless stated otherwise. The
 *    caller owns every buffer, the workspace and the stream; the library
 *    allocates no memory and keeps no state besides a thread-local error
 *    message (and the fixed device array of nsnq_attn_decode_noalloc). Calls are asynchronous on `stream` (NULL = legacy default
 *    stream) and never synchronise.
 *  - Arguments are validated on the host before anything is launched; on
 *    error the call returns a non-zero status, writes nothing, launches
 *    nothing, and nsnq_last_error() describes the problem. A failed launch
 *    returns NSNQ_ERR_CUDA. Faults that happen later on the device surface on
 *    the stream like any CUDA error.
 *  - Supported: D = 128, 256 centroids, sub_dim in {4, 8}, Hq % Hkv == 0.
 *    Query head h reads kv-head h / (Hq / Hkv).
 *  - Cache layout (one nsnq_cache per tensor, K and V separately):
 *      codes  uint8 [B][H][cap][D/sub_dim], sub-vector j ascending
 *      scales fp32  [B][H][cap][2] = (s1, s2)
 *      shift  fp32  [B][H][D]      = o
 *    or, for double-quantized byproducts stored packed (s1_levels != NULL):
 *      scales    fp32   [B][H][cap]         = s2 (sign bit set: s1 = 0)
 *      s1_levels uint32 [B][H][(cap+7)/8]   4-bit s1 level of token t in
 *                                           bits 4(t%8)..4(t%8)+3 of word t/8
 *      s1_grid   fp32   [B][H][2]           = (lo, step): level k means
 *                                           s1 = 2^(lo + k step), evaluated in
 *                                           fp64 and rounded to fp32
 */
#ifndef NSNQ_H_
#define NSNQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the runtime's stream handle); NULL is the legacy default stream. */
typedef struct CUstream_st* nsnq_stream;

typedef enum {
    NSNQ_OK = 0,
    NSNQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, stride or range */
    NSNQ_ERR_UNSUPPORTED = 2,  /* valid but not implemented (D != 128, sub_dim, ...) */
    NSNQ_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    NSNQ_ERR_CUDA = 4          /* a CUDA call or kernel launch failed */
} nsnq_status;

typedef enum { NSNQ_F32 = 0, NSNQ_BF16 = 1 } nsnq_dtype;

typedef enum {
    NSNQ_SHIFT_COMPUTE = 0,  /* o = mean of the normalized tokens of this call (a prompt) */
    NSNQ_SHIFT_GIVEN = 1     /* o read from cache.shift (tokens appended after the prompt) */
} nsnq_shift_mode;

typedef enum {
    NSNQ_ENCODE_DEFAULT = 0,
    /* Scale adjustment (Methodology §3): the quantized token w_hat is scaled by
     * ||w||^2 / (w . w_hat) so that its component along the transformed token w
     * equals w (the error left is orthogonal to w); the factor multiplies the
     * stored s2, so dequant and attention need no change. */
    NSNQ_ENCODE_ADAPTIVE_SCALE = 1,
    /* Double quantization (Methodology §3): s1 takes one of 16 levels of a
     * per-head grid uniform in log2 (grid = (lo, step), from the least to
     * the largest log2 s1 of the tokens encoded in shift-compute mode, kept
     * in cache.s1_grid for later shift-given appends), and a computed o takes
     * one of 16 uniform levels between its least and largest channel value.
     * With cache.s1_levels == NULL the level values go to the usual fp32
     * fields; with cache.s1_levels set, s1 is stored as its 4-bit level and
     * scales holds s2 alone (the packed form, see nsnq_cache). o stays an
     * fp32 vector per head (its 16 level values). Requires cache.s1_grid. */
    NSNQ_ENCODE_DOUBLE_QUANT = 2,
    /* sub_dim 4: find the nearest codeword by scoring all 256 on the tensor
     * cores (|C|^2 - 2 w.C, as for sub_dim 8) instead of walking the search
     * index; cb.index is then not needed. Same codes (exact up to the
     * near-tie rule), slower than the index walk: it serves codebooks whose
     * index does not fit (nsnq_codebook_index_build returns
     * NSNQ_ERR_UNSUPPORTED) and comparison. Calls of at most 1024
     * token-heads use the small-call path either way. No effect at sub_dim 8. */
    NSNQ_ENCODE_TC_SEARCH = 4
} nsnq_encode_flags;

typedef struct {
    const float* centroids;  /* device, [n_centroids][sub_dim] fp32, 16-byte aligned */
    int n_centroids;         /* must be 256 (one byte per code) */
    int sub_dim;             /* 4 (2 bits/coordinate) or 8 (1 bit/coordinate) */
    const void* index;       /* device search index built from these centroids by
                                nsnq_codebook_index_build; required by nsnq_encode when
                                sub_dim == 4 unless NSNQ_ENCODE_TC_SEARCH is passed,
                                ignored otherwise (may be NULL) */
} nsnq_codebook;

typedef struct {
    uint8_t* codes;   /* device, [B][H][cap][D/sub_dim] */
    float* scales;    /* device, [B][H][cap][2] = (s1, s2) */
    float* shift;     /* device, [B][H][D] = o */
    int64_t cap;      /* token capacity per (batch, head) */
    float* s1_grid;   /* device, [B][H][2] = (lo, step) of the double-quantized s1 grid
                         (log2 domain), or NULL without double quantization */
    uint32_t* s1_levels; /* device, [B][H][(cap+7)/8], or NULL. Non-NULL selects the packed
                         double-quantized form (Methodology §3, Double Quantization: s1
                         takes 4 bits): s1 is kept only as its 4-bit level on the head's
                         grid (s1_grid, required), and scales holds s2 alone,
                         [B][H][cap] fp32; a token with s1 = 0 (an all-zero token) has
                         level 0 and the sign bit of its stored s2 set. Per token-head this
                         stores 4.5 bytes of byproducts instead of 8. Only encode calls
                         with NSNQ_ENCODE_DOUBLE_QUANT may write a packed cache; dequant
                         and the attention calls read either form. 4-byte aligned. */
} nsnq_cache;

/* Human-readable name of a status code (static string). */
const char* nsnq_status_string(nsnq_status status);

/* Detail of the last error returned on the calling thread ("" if none). */
const char* nsnq_last_error(void);

/*
 * Bytes of the nearest-codeword search index of a sub_dim = 4 codebook
 * (0 for sub_dim = 8, which needs none).
 */
size_t nsnq_codebook_index_bytes(int sub_dim);

/*
 * nsnq_codebook_index_build -- one-time preparation of a 2-bit codebook for
 * nsnq_encode (no counterpart on the pages: it accelerates the exact
 * nearest-codeword search of Methodology §3). Each coordinate of the
 * transformed sub-vector is binned on a fixed grid; for every grid cell the
 * index lists, sorted by a lower bound of their distance over the cell, the
 * codewords that can be nearest (or within the near-tie band of the
 * nearest) somewhere in the cell. cb.index is ignored; on success set
 * cb.index = index for later calls. `index` must hold
 * nsnq_codebook_index_bytes(4) bytes (16-byte aligned). This call waits for
 * `stream` to finish (it checks that the lists fit) and returns
 * NSNQ_ERR_UNSUPPORTED if they do not.
 */
nsnq_status nsnq_codebook_index_build(nsnq_codebook cb, void* index, size_t index_bytes,
                                      nsnq_stream stream);

/*
 * nsnq_codebook_quantize4 -- the double-quantized form of a codebook
 * (Methodology §3, Double Quantization: the codebook entries take 4-bit
 * values). All n_centroids * sub_dim entries share one grid of 16 uniform
 * levels from their least value lo to their largest value hi:
 * step = (hi - lo) / 15 and entry e becomes lo + k * step with
 * k = (e - lo) / step rounded to the nearest integer (halves away from
 * zero), computed in fp64 and rounded to fp32 (k = 0 for every entry when
 * hi == lo).
 *   centroids  device [n_centroids][sub_dim] fp32 (n_centroids 256, sub_dim 4 or 8).
 *   out        device, same shape: the level values; may equal centroids.
 *   levels     device [n_centroids * sub_dim / 2] bytes or NULL: the 4-bit k
 *              of entry i in byte i / 2 (even i in the low nibble).
 *   grid       device double[2] = (lo, step) or NULL.
 * The result is a codebook like any other: pass `out` as the centroids of
 * nsnq_encode (build the index from it for sub_dim 4), nsnq_dequant and the
 * attention calls. Asynchronous on `stream`.
 */
nsnq_status nsnq_codebook_quantize4(const float* centroids, float* out, uint8_t* levels,
                                    double* grid, int n_centroids, int sub_dim,
                                    nsnq_stream stream);

/*
 * Workspace bytes nsnq_encode needs for this shape (any shift mode). The
 * first 64 bytes hold counters the call resets and fills:
 *   uint64 [0] token-heads re-encoded on the fp64 near-tie path,
 *   uint64 [1] sub-vectors whose code was decided on that path,
 *   uint64 [2] nonzero if cb.index was not built from cb.centroids,
 *   uint64 [3] used internally (work counter),
 *   uint64 [4] nonzero if a tensor-core scoring round (sub_dim 8, or 4 with
 *              NSNQ_ENCODE_TC_SEARCH) was not
 *              seen complete within its bounded wait: the CTA that waited
 *              stopped, so some codes and scales of this call are NOT
 *              written and the call's result is void. The status returned
 *              by nsnq_encode cannot report it (the kernel runs after the
 *              call returns): read this word after the stream has finished.
 */
size_t nsnq_encode_workspace(int B, int H, int64_t T, int D);

/*
 * nsnq_encode -- NSN normalize/shift/normalize, Hadamard transform and
 * nearest-codeword quantization of T tokens per (batch, head)
 * (Methodology §1-§3), written to cache positions [t_offset, t_offset+T).
 *
 *   x         device, element (b, h, t, c) at x[b*stride_b + h*stride_h +
 *             t*stride_t + c] (strides in elements, channels contiguous),
 *             dtype x_dtype (fp32 or bf16); 16-byte aligned rows.
 *   mode      NSNQ_SHIFT_COMPUTE: o = mean over the T tokens of x/s1, stored
 *             to cache.shift (fp32); NSNQ_SHIFT_GIVEN: o = cache.shift.
 *   flags     NSNQ_ENCODE_DEFAULT, or any of NSNQ_ENCODE_ADAPTIVE_SCALE,
 *             NSNQ_ENCODE_DOUBLE_QUANT, NSNQ_ENCODE_TC_SEARCH (bitwise or);
 *             other bits: NSNQ_ERR_INVALID_ARG.
 *   cb        codebook; cache: codes/scales written, shift read or written.
 *   workspace device scratch of at least nsnq_encode_workspace(B, H, T, D)
 *             bytes, 256-byte aligned.
 * Codes equal the nearest codeword of the exact (fp64) transformed token;
 * sub-vectors whose two best fp32 distances are within the near-tie band
 * (a bound on the fp32 / three-term tf32 scoring error) are re-decided in
 * fp64. Calls of at most 1024 token-heads (B*H*T, e.g. a decode step's
 * appends) take a one-warp-per-token-head path instead: NSN and the
 * Hadamard transform in fp64, an fp32 scan of all 256 codewords keeping the
 * best and second best, and an fp64 re-scan of the sub-vectors inside the
 * near-tie band; the index is not read and the workspace counters stay 0.
 * Stored s1, s2, o are fp32 roundings. A zero-norm token (or a zero residual after the shift) maps to
 * the zero vector with s = 0. T = 0 is a no-op. At most 2^31 - 1 token-heads
 * (B*H*T) per call: NSNQ_ERR_UNSUPPORTED above.
 */
nsnq_status nsnq_encode(const void* x, nsnq_dtype x_dtype, int B, int H, int64_t T, int D,
                        int64_t stride_b, int64_t stride_h, int64_t stride_t, int64_t t_offset,
                        nsnq_shift_mode mode, unsigned flags, nsnq_codebook cb, nsnq_cache cache,
                        void* workspace, size_t workspace_bytes, nsnq_stream stream);

/*
 * nsnq_encode_kv -- nsnq_encode of a layer's keys and values in one call.
 * NSNQuant quantizes both caches with one global codebook (Methodology §3),
 * so the two tensors can share every launch of the call: one index staging,
 * one work queue over the token-heads of both, and no idle tail between
 * them. Each argument means what it means for nsnq_encode, applied to
 * (x_k, cache_k) and to (x_v, cache_v); the two tensors share dtype, shape,
 * strides, t_offset, mode, flags and the codebook, and the caches must agree
 * in cap and form (both packed or neither) and share no buffer (the same
 * codes, scales, shift, s1_levels or s1_grid pointer: NSNQ_ERR_INVALID_ARG;
 * overlapping views of one allocation are the caller's to avoid). Codes, s1, s2 and o carry the
 * guarantees of nsnq_encode for each tensor; the fp64 channel sums behind o
 * are grouped by this call's chunk plan, so o can differ in its last fp32
 * bit from a separate nsnq_encode of the same tensor. The workspace counters
 * count both tensors.
 *   workspace  >= nsnq_encode_kv_workspace(B, H, T, D) bytes (that of
 *              nsnq_encode at batch 2B), 256-byte aligned.
 * B <= 32767 and 2*B*H*T < 2^31 (NSNQ_ERR_UNSUPPORTED above); T = 0 is a
 * no-op.
 */
size_t nsnq_encode_kv_workspace(int B, int H, int64_t T, int D);
nsnq_status nsnq_encode_kv(const void* x_k, const void* x_v, nsnq_dtype x_dtype, int B, int H,
                           int64_t T, int D, int64_t stride_b, int64_t stride_h, int64_t stride_t,
                           int64_t t_offset, nsnq_shift_mode mode, unsigned flags, nsnq_codebook cb,
                           nsnq_cache cache_k, nsnq_cache cache_v, void* workspace,
                           size_t workspace_bytes, nsnq_stream stream);

/*
 * nsnq_dequant -- reconstruct tokens [t0, t0+T) of every (batch, head):
 * out = s1 * (s2 * H w_hat + o), w_hat the concatenated codewords
 * (Methodology §1: the byproducts reconstruct the tensor).
 *   out  device fp32 [B][H][T][D], 16-byte aligned.
 * No workspace. T = 0 is a no-op.
 */
nsnq_status nsnq_dequant(nsnq_cache cache, nsnq_codebook cb, int B, int H, int64_t t0, int64_t T,
                         int D, float* out, nsnq_stream stream);

/* Workspace bytes nsnq_attn_decode needs (split-context partials). */
size_t nsnq_attn_workspace(int B, int Hq, int Hkv, int D, int64_t max_len);

/*
 * nsnq_attn_decode -- one decode step of attention for one query token per
 * sequence, reading the quantized K/V caches directly (Methodology §4):
 *   score_t = scale * q . k_hat_t
 *           = scale * s1_t * (s2_t * sum_j L[j][code_t,j] + q . o_K),
 *     L[j][c] = (H q)[j*g:(j+1)*g] . C_c   (H symmetric, so q . H w = (Hq) . w),
 *   out = sum_t softmax(score)_t v_hat_t
 *       = (H sum_t p_t s1_t s2_t w_hat_t + (sum_t p_t s1_t) o_V) / sum_t p_t.
 *   q        device [B][Hq][D], q_dtype (fp32 or bf16).
 *   k_cache, v_cache, k_cb, v_cb: caches and their codebooks (sub_dims may differ).
 *   seq_lens device int32 [B]; sequence b attends to its first
 *            min(seq_lens[b], max_len) tokens (0 gives a zero output).
 *   max_len  host upper bound on seq_lens, <= both caps; sizes the split plan.
 *   softmax_scale  0 means 1/sqrt(D).
 *   out      device [B][Hq][D], out_dtype (fp32 or bf16, rounded to nearest even).
 *   workspace  >= nsnq_attn_workspace(B, Hq, Hkv, D, max_len) bytes, 256-byte aligned.
 */
nsnq_status nsnq_attn_decode(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                             nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                             const int32_t* seq_lens, int64_t max_len, int B, int Hq, int Hkv,
                             int D, float softmax_scale, void* out, nsnq_dtype out_dtype,
                             void* workspace, size_t workspace_bytes, nsnq_stream stream);

/*
 * Full-precision residual window (Methodology §4, Implementation Details,
 * Residuals): the most recent tokens of each sequence, kept unquantized
 * until the window fills; then they are quantized (nsnq_encode with
 * NSNQ_SHIFT_GIVEN on the window, t_offset = the sequence's quantized
 * length) and the window is emptied.
 */
typedef struct {
    const void* k;        /* device [B][Hkv][cap][D] of dtype, 16-byte aligned */
    const void* v;        /* device [B][Hkv][cap][D] of dtype, 16-byte aligned */
    nsnq_dtype dtype;     /* NSNQ_F32 or NSNQ_BF16 */
    const int32_t* lens;  /* device int32 [B]: residual tokens of sequence b */
    int64_t cap;          /* rows per (batch, kv-head) */
} nsnq_residual;

/*
 * nsnq_attn_decode_res -- nsnq_attn_decode over the first seq_lens[b]
 * quantized tokens followed by the first min(max(res.lens[b], 0), res.cap)
 * residual tokens of each sequence, one softmax over both:
 *   out = (H A + beta o_V + sum_r p_r v_r) / (sum_t p_t + sum_r p_r),
 * residual scores scale * q . k_r in fp32 from the stored K rows.
 * res.cap = 0 (pointers may then be NULL) is exactly nsnq_attn_decode.
 * A sequence with no token at all gets a zero output. Other arguments,
 * the workspace and the errors are those of nsnq_attn_decode.
 */
nsnq_status nsnq_attn_decode_res(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                                 nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                                 const int32_t* seq_lens, int64_t max_len, nsnq_residual res,
                                 int B, int Hq, int Hkv, int D, float softmax_scale, void* out,
                                 nsnq_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                 nsnq_stream stream);

/*
 * nsnq_residual_write -- copy T tokens of every (batch, head) into rows
 * [t_offset, t_offset + T) of a residual buffer buf [B][H][cap][D] of
 * buf_dtype, converting (fp32 to bf16 rounds to nearest even; the other
 * directions are exact). x is laid out as for nsnq_encode. The rows must
 * fit: 0 <= t_offset and t_offset + T <= cap. T = 0 is a no-op.
 */
nsnq_status nsnq_residual_write(const void* x, nsnq_dtype x_dtype, int B, int H, int64_t T, int D,
                                int64_t stride_b, int64_t stride_h, int64_t stride_t,
                                int64_t t_offset, void* buf, nsnq_dtype buf_dtype, int64_t cap,
                                nsnq_stream stream);

/*
 * nsnq_attn_decode_rope -- nsnq_attn_decode for keys quantized before the
 * rotary position embedding (Methodology §4, Implementation Details: NSN is
 * applied to the keys before RoPE). Key t of a sequence (cache position t)
 * is dequantized, k_t = s1 (s2 H w_hat + o), rotated to position t and
 * dotted with q, which the caller passes already rotated at its own
 * position:
 *   (k_i, k_{i+D/2}) -> (k_i c - k_{i+D/2} s, k_i s + k_{i+D/2} c),
 *   c, s = cos, sin of t * rope_base^(-2i/D), i < D/2.
 *   rope_base  finite, > 1 (10000 in most models).
 * Values, workspace (nsnq_attn_workspace), outputs and errors are those of
 * nsnq_attn_decode; there is no residual window here.
 */
nsnq_status nsnq_attn_decode_rope(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                                  nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                                  const int32_t* seq_lens, int64_t max_len, double rope_base,
                                  int B, int Hq, int Hkv, int D, float softmax_scale, void* out,
                                  nsnq_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                  nsnq_stream stream);

/*
 * nsnq_attn_decode_noalloc -- nsnq_attn_decode for callers that cannot
 * allocate device memory (no workspace argument). The method has no
 * counterpart for this: it is a packaging of the same kernels.
 *
 * Who needs it: code that cannot call cudaMalloc or reach an allocator --
 * a plugin inside an engine that owns all device memory, a real-time loop
 * where an allocation (which may synchronise the device) is not allowed, or
 * a C caller without an allocator. The caller still passes q, the caches,
 * seq_lens and out; only the split-context partials move into a fixed
 * 4 MiB array in device global memory that the library defines. Every GPU
 * that loads the library reserves those 4 MiB until the process exits.
 *
 * Limit: shapes whose partials need more than 4 MiB
 * (nsnq_attn_workspace(B, Hq, Hkv, D, max_len) > 4194304) are rejected with
 * NSNQ_ERR_WORKSPACE before anything is launched.
 * Every call whose `stream` is not capturing looks up the array's device
 * address on the current device (cudaGetSymbolAddress), so the entry point
 * stays valid after cudaDeviceReset, which can move the array. Make the
 * first call on each device before any stream capture: a first call on a
 * capturing stream returns NSNQ_ERR_INVALID_ARG. The array is shared by all calls and keeps the
 * last call's contents; nothing in it needs to start at zero. Calls that
 * overlap on the GPU (different streams, or different host threads on the
 * same device) race on the array: serialise them. Arguments, errors and
 * results are otherwise exactly those of nsnq_attn_decode.
 */
nsnq_status nsnq_attn_decode_noalloc(const void* q, nsnq_dtype q_dtype, nsnq_cache k_cache,
                                     nsnq_cache v_cache, nsnq_codebook k_cb, nsnq_codebook v_cb,
                                     const int32_t* seq_lens, int64_t max_len, int B, int Hq,
                                     int Hkv, int D, float softmax_scale, void* out,
                                     nsnq_dtype out_dtype, nsnq_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* NSNQ_H_ */
