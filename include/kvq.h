/*
 * kvq.h -- C ABI of libkvq: attention over a block-quantized, mixed-precision KV cache
 * on NVIDIA B200 (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *   [KVBENCH]  "KV cache quant benchmarks: KVarN 6-bit matches q8_0, 4-bit matches q5_0"
 *              -- cache-size column of the KLD table (block byte counts).
 *   [HARDNUM]  "Hard numbers on Qwen3.8-27B's KV cache: q8_0 is free, K is ~2x as touchy as
 *              V, and a 2k recent-token window makes 6/5-bit basically lossless"
 *              -- "KV cache low-bit storage" (config D: K 6-bit, V 5-bit, last 2,048
 *              positions in an 8-bit ring) and "Reddit reactions" (two KV paths per layer,
 *              requantization when the window boundary moves; 32 values per token block).
 *   [BEELLAMA] "BeeLlama.cpp v0.4.1: KVarN, KV precision tail, q2_0-q3_1 KV cache"
 *              -- KVarN, the bf16/f16 precision tail, the q2/q3/q6 types, KV-MiB table.
 *   [OFFLOAD]  "You can offload most of Qwen3.8-Flash-Next's KV cache to RAM with little
 *              decode slowdown" -- decode is bound by the bytes each step reads.
 *
 * Conventions for every entry point:
 *  - Pointers named dev_* / k / v / q / out / ws are DEVICE pointers (cudaMalloc or torch
 *    memory on the cache's device), 16-byte aligned, row-major, float32 unless stated.
 *    host_* pointers are host memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Calls
 *    that launch work are asynchronous on that stream; one cache handle must be used
 *    from one stream at a time.
 *  - The caller owns all device memory: the cache buffer, inputs, outputs and
 *    workspace. The library owns only the host-side descriptor and allocates no
 *    device memory.
 *  - Every call returns a kvq_status. Arguments are validated on the host before
 *    anything is launched: a failed call launches nothing, writes nothing and leaves
 *    the cache length unchanged. Launch failures are reported as KVQ_ERR_CUDA.
 *    Nothing throws across the ABI and nothing aborts the process.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1,     /* bad pointer, shape, index or option */
    KVQ_ERR_UNSUPPORTED_FMT = 2, /* format not allowed in that role */
    KVQ_ERR_CAPACITY = 3,        /* append beyond max_ctx */
    KVQ_ERR_CALIBRATION = 4,     /* KVarN: first append shorter than the calibration window */
    KVQ_ERR_EMPTY = 5,           /* attention over an empty cache */
    KVQ_ERR_ALIGNMENT = 6,       /* a device pointer is not 16-byte aligned */
    KVQ_ERR_NOT_BOUND = 7,       /* no device buffer bound yet */
    KVQ_ERR_CUDA = 8,            /* a CUDA runtime call or launch failed */
    KVQ_ERR_DEVICE_TIMEOUT = 9   /* a kernel gave up a bounded device-side wait (see kvq_device_status) */
} kvq_status;

/* Block formats. A block is 32 consecutive channels of one token row ([HARDNUM],
 * "Reddit reactions": 32 values grouped per token).
 *  qX_0: fp16 scale d + 32 X-bit codes, 2 + 4X bytes; value = d * (u - 2^(X-1)),
 *        d = fp16(absmax / (2^(X-1) - 1)), codes round half away from zero, then clamp.
 *  qX_1: fp16 scale d + fp16 min m + 32 X-bit codes, 4 + 4X bytes; value = d * u + m,
 *        d = fp16((max - min) / (2^X - 1)), m = fp16(min).
 *  Byte counts match [KVBENCH] (q8_0 34/64 of bf16, q6_0 26/64, q5_1 24/64) and the
 *  [BEELLAMA] KV-MiB table. BF16 / F16 store 16-bit floats (tail formats only). */
typedef enum kvq_fmt {
    KVQ_Q2_0 = 0, KVQ_Q2_1 = 1, KVQ_Q3_0 = 2, KVQ_Q3_1 = 3,
    KVQ_Q4_0 = 4, KVQ_Q4_1 = 5, KVQ_Q5_0 = 6, KVQ_Q5_1 = 7,
    KVQ_Q6_0 = 8, KVQ_Q6_1 = 9, KVQ_Q8_0 = 10, KVQ_Q8_1 = 11,
    KVQ_BF16 = 12, KVQ_F16 = 13, KVQ_NONE = 14
} kvq_fmt;

/* Shape of a cache. head_dim in {32, 64, 128, 256}; n_q_heads = G * n_kv_heads with
 * 1 <= G <= 8; query head hq reads KV head hq / G. kvarn = 1 enables variance-normalised
 * blocks ([BEELLAMA] names KVarN): per (layer, batch, kv head, channel, K|V)
 * s = fp32(sqrt(S / T + eps)), S the fp64 sum of x^2 over the first T =
 * kvarn_calib_tokens tokens (a power of two, 64..1024) taken as a fixed pairwise tree;
 * blocks store x / s and are read back as s * value.
 * k_per_channel = 1 quantizes K along the token axis ([HARDNUM] "Reddit reactions": the KIVI
 * question; per-channel K reduced the error without a window and did not beat per-token blocks
 * with the 2k window): a K block holds 32 consecutive positions of one channel, quantized with
 * the same rules when the last of them enters the K store; positions that entered before
 * their group is complete are kept exactly (float32) until it is. V keeps per-token blocks.
 * Not combined with kvarn. Attention over such a cache runs on the CUDA-core path. */
typedef struct kvq_layout {
    int32_t n_layers;
    int32_t batch;
    int32_t n_kv_heads;
    int32_t n_q_heads;
    int32_t head_dim;
    int32_t kvarn;               /* 0 or 1 */
    int64_t max_ctx;             /* positions per (layer, batch element) */
    int32_t kvarn_calib_tokens;  /* 512 by convention */
    int32_t k_per_channel;       /* 0: K blocks of 32 channels of a token; 1: K blocks of 32
                                    positions of a channel (see below) */
    double kvarn_eps;            /* 1e-6 by convention */
} kvq_layout;

typedef struct kvq_cache kvq_cache;

/* Create a host-side cache descriptor. k_fmt, v_fmt: any qX_0 / qX_1 format.
 * tail_fmt: KVQ_NONE (W must be 0) or KVQ_Q8_0 / KVQ_BF16 / KVQ_F16 with W >= 1: the
 * most recent W positions are kept in that format in a W-row ring and requantized to
 * the low-bit format when they leave the window ([HARDNUM] "KV cache low-bit storage",
 * [BEELLAMA] precision tail). kvarn with a tail: the ring holds raw values and the
 * normalisation is applied at requantization. *out receives the handle. */
KVQ_API kvq_status kvq_cache_create(const kvq_layout* layout, kvq_fmt k_fmt, kvq_fmt v_fmt,
                            kvq_fmt tail_fmt, int32_t W, kvq_cache** out);

/* Bytes of device memory the cache needs ([BEELLAMA] KV-MiB table and [KVBENCH] cache-size
 * column: the store is max_ctx rows of the block format per layer, kv head, K and V; the
 * precision tail adds W rows of the tail format on top): the low-bit store, the ring, the
 * KVarN scales and a metadata region of 256 + 16 * n_layers * batch * n_kv_heads bytes
 * rounded up to 256 (a device status word and per-head value bounds). Without the
 * metadata region this equals the block-size closed form when every row is a multiple of
 * 16 bytes and max_ctx, W are multiples of 16 (rows are otherwise padded to 16 bytes,
 * regions to 256). */
KVQ_API kvq_status kvq_cache_required_bytes(const kvq_cache* cache, size_t* bytes);

/* Bind caller-owned device memory (>= required bytes, 256-byte aligned) on the current
 * device: the memory holds the rows [OFFLOAD] sizes per token and layer (row-size
 * paragraph) in the block formats above. Zero-fills it on `stream` and resets every
 * layer's length to 0. Also maps the fixed array of kvq_decode_attention_noalloc on this
 * device (looked up once per device). KVQ_ERR_CUDA if a CUDA call fails. */
KVQ_API kvq_status kvq_cache_bind(kvq_cache* cache, void* dev_buf, size_t bytes, void* stream);

/* Free the host descriptor (never the bound device memory). NULL is accepted. Nothing on
 * the pages corresponds to it; it ends the descriptor's lifetime. */
KVQ_API kvq_status kvq_cache_destroy(kvq_cache* cache);

/* Quantize-on-append of n_new positions to layer `layer` (all batch elements)
 * ([HARDNUM] "Reddit reactions": each token row is quantized in 32-value blocks as it
 * enters, and blocks are requantized when the window boundary moves; "KV cache low-bit
 * storage": the last 2,048 positions stay in the 8-bit ring).
 * k, v: float32 [batch][n_new][n_kv_heads][head_dim]. Positions n..n+n_new-1 are
 * written: those that end inside the window go to the ring in tail format (evicting
 * and requantizing the positions they displace), the others straight to the low-bit
 * store (with a tail: through the tail format first, so chunking never changes the
 * stored bytes). With kvarn and no scales set, the first append must carry at least
 * kvarn_calib_tokens positions (KVQ_ERR_CALIBRATION otherwise) and computes the
 * scales from them first. n_new = 0 is a no-op. */
KVQ_API kvq_status kvq_append(kvq_cache* cache, int32_t layer, const float* k, const float* v,
                      int32_t n_new, void* stream);

/* Workspace bytes for kvq_decode_attention (n_query_rows = 1) or kvq_prefill_attention
 * (n_query_rows = n_chunk). For a prefill at head dim 128 / 256 with n_chunk * G > 128 (more
 * than one 128-row tile of query rows per kv head) the workspace holds the K~ / V~ operand
 * tiles dequantized once per (batch, kv head): 128 * head_dim bytes per position of max_ctx
 * per (batch, kv head), then room for up to 4 key-range partials of every query row
 * (4 * batch * n_chunk * n_q_heads * (head_dim + 2) floats; the library splits the rows'
 * key range when that fills the GPU better, and merges the partials). With a single tile
 * per kv head (n_chunk * G <= 128, n_chunk > 1) it holds up to 64 such partials per row, or
 * the split-K partials below if those are larger. Otherwise it holds the per-split softmax partials of the
 * split-K decode ([OFFLOAD]: decode streams the whole attention state each step, so the
 * positions are split across the GPU and the partials merged). KVQ_ERR_NOT_BOUND before a
 * bind (the split count depends on the device's SM count). */
KVQ_API kvq_status kvq_decode_workspace_bytes(const kvq_cache* cache, int32_t n_query_rows, size_t* bytes);

/* Decode attention (GQA) over all n cached positions of `layer` ([OFFLOAD] decode-is-
 * bandwidth paragraph: each step reads every cached row; [HARDNUM] "KV cache low-bit
 * storage": the low-bit rows plus the 8-bit recent-token ring of config D):
 * out[b][hq] = softmax_t(scale * q[b][hq] . K~[b][hq/G][t]) . V~[b][hq/G][t], with K~, V~
 * the dequantized cache (ring rows for the last min(n, W) positions). q, out: float32
 * [batch][n_q_heads][head_dim]. Split-K over positions, then a fixed-order merge, so the
 * result is bit-reproducible. ws: device workspace of >= kvq_decode_workspace_bytes(1).
 * KVQ_ERR_EMPTY when n = 0. */
KVQ_API kvq_status kvq_decode_attention(kvq_cache* cache, int32_t layer, const float* q, float scale,
                                float* out, void* ws, size_t ws_bytes, void* stream);

/* Index-gather decode ([OFFLOAD], the QSA paragraph: an indexer picks a budget of 2,048
 * positions per step and attention reads only those rows of the quantized cache): like
 * kvq_decode_attention, but each (batch element, kv head) attends only to the positions
 * it lists. idx: device int32 [batch][n_kv_heads][n_idx], 4-byte aligned, 1 <= n_idx <=
 * KVQ_MAX_GATHER. Entries outside [0, n) are skipped; the others enter the softmax in list
 * order, a repeated position counting once per entry; a list without a valid entry gives a
 * zero output. Rows are fetched by one bulk copy each from the low-bit store or the ring,
 * wherever the position lies. ws: >= kvq_decode_workspace_bytes(cache, 1). */
#define KVQ_MAX_GATHER 65536
KVQ_API kvq_status kvq_decode_attention_indexed(kvq_cache* cache, int32_t layer, const float* q, float scale,
                                        const int32_t* idx, int32_t n_idx, float* out, void* ws,
                                        size_t ws_bytes, void* stream);

/* Causal chunked-prefill attention for the n_chunk positions just appended ([HARDNUM]
 * "Engine speed and cache reuse": prompt processing with the config D cache; chunk row i
 * sits at position n - n_chunk + i and attends to positions <= its own over the
 * post-append cache). q, out: float32 [batch][n_chunk][n_q_heads][head_dim].
 * Requires 1 <= n_chunk <= n. ws: >= kvq_decode_workspace_bytes(n_chunk). Chunks of up to 4
 * rows (a multi-query verify) run on the split-K decode kernels, one pass over the keys per
 * row; longer chunks at head dim 128 / 256 on the tensor-core (tcgen05) prefill, which may
 * split each 128-row tile of query rows over the key range and merge the parts. */
KVQ_API kvq_status kvq_prefill_attention(kvq_cache* cache, int32_t layer, const float* q, int32_t n_chunk,
                                 float scale, float* out, void* ws, size_t ws_bytes, void* stream);

/* Decode attention exactly as kvq_decode_attention, but without a caller workspace and
 * without allocating anything: the softmax partials go to a fixed array of
 * KVQ_NOALLOC_WORKSPACE_MIB MiB inside the library's device image. For callers that
 * cannot call cudaMalloc or pass a workspace (e.g. a plugin inside a host program that
 * owns the device allocator, or a C caller whose device footprint must stay fixed after
 * start-up). The pages have no counterpart to this entry point; it is a deployment aid.
 *  - Every GPU that loads the library holds the array until the process exits.
 *  - The array's device address is looked up (cudaGetSymbolAddress) once per device, when
 *    a cache is first bound on it (kvq_cache_bind) or at the first call on it, with that
 *    device current; with CUDA's lazy module loading that lookup is also when the array
 *    is mapped. Make that first bind or call before any stream capture.
 *  - The cache's device must be the current device (KVQ_ERR_INVALID_ARG otherwise).
 *  - A cache whose decode needs more workspace than the array holds
 *    (kvq_decode_workspace_bytes(cache, 1) > KVQ_NOALLOC_WORKSPACE_MIB MiB) is rejected
 *    with KVQ_ERR_CAPACITY before anything is launched.
 *  - All calls share the array and it keeps the last call's contents (nothing in it has
 *    to start at zero). Calls whose kernels overlap on the GPU race on it: issue them on
 *    one stream, one after another.
 * Calls no cudaMalloc, cudaFree or allocating routine. */
#define KVQ_NOALLOC_WORKSPACE_MIB 8
KVQ_API kvq_status kvq_decode_attention_noalloc(kvq_cache* cache, int32_t layer, const float* q, float scale,
                                        float* out, void* stream);

/* Current number of cached positions of `layer` (host-tracked, uniform over batch): the
 * context length n of [HARDNUM] "KV cache low-bit storage", which decides which positions
 * are in the recent-token ring (the last min(n, W)). */
KVQ_API kvq_status kvq_length(const kvq_cache* cache, int32_t layer, int64_t* n);

/* KVarN only ([BEELLAMA] KVarN paragraph: variance-normalised blocks): set the channel
 * scales of `layer` instead of calibrating. sK, sV: device float32
 * [batch][n_kv_heads][head_dim], all > 0. Must come before the layer's first append. */
KVQ_API kvq_status kvq_set_channel_scales(kvq_cache* cache, int32_t layer, const float* sK, const float* sV,
                                  void* stream);

/* KVarN only ([BEELLAMA] KVarN paragraph): copy the channel scales of `layer` (calibrated
 * or set) to host memory. host_sK, host_sV: float32 [batch][n_kv_heads][head_dim].
 * Synchronises the device. KVQ_ERR_CALIBRATION if the layer has no scales yet. */
KVQ_API kvq_status kvq_get_channel_scales(const kvq_cache* cache, int32_t layer, float* host_sK, float* host_sV);

/* Device status of the cache. Every wait a kernel makes on the device (a pipeline barrier)
 * is bounded; a wait that runs out makes the kernel stop waiting, poison its output with NaN
 * and record the event in a status word inside the bound buffer. This call synchronises
 * `stream`, reads the word and clears it: KVQ_OK if no wait ran out since the last call,
 * KVQ_ERR_DEVICE_TIMEOUT otherwise. The pages have no counterpart; it is the failure
 * report of the pipelined kernels. */
KVQ_API kvq_status kvq_device_status(kvq_cache* cache, void* stream);

/* Check of the failure path above: one warp waits, with the same bounded wait the
 * pipelined kernels use and a limit of limit_ns (<= 10 s), on a barrier that nothing
 * arrives on, then records the timeout in the cache's status word (kvq_device_status then
 * returns KVQ_ERR_DEVICE_TIMEOUT). Holds no copies or tensor memory. Asynchronous on
 * `stream`. The pages have no counterpart. */
KVQ_API kvq_status kvq_selftest_wait_timeout(kvq_cache* cache, uint64_t limit_ns, void* stream);

/* Copy stored rows to host memory in the canonical serialisation of [KVBENCH] /
 * [BEELLAMA] block byte counts. With k_per_channel, K region 0 copies groups pos0 ..
 * pos0 + count - 1 (each D canonical blocks in channel order) and K region 2 copies pending
 * slots pos0 .. (float32 rows of head_dim values, pos0 + count <= 32). Otherwise (per 32-value
 * block:
 * fp16 d | [fp16 m] | code planes low bits first, little endian; BF16/F16: 32 x 2 bytes).
 * region 0: low-bit store rows pos0..pos0+count-1; region 1: ring slots pos0..+count-1
 * (tail format). kv: 0 = K, 1 = V. Synchronises the device. host_dst must hold
 * count * (head_dim / 32) * block bytes. */
KVQ_API kvq_status kvq_export_blocks(const kvq_cache* cache, int32_t layer, int32_t b, int32_t h, int32_t kv,
                             int32_t region, int64_t pos0, int64_t count, void* host_dst, size_t bytes);

/* Static description of a status code (no counterpart on the pages). */
KVQ_API const char* kvq_status_string(kvq_status status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
