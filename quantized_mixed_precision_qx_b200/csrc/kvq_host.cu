// kvq_host.cu -- the C ABI of libkvq: cache descriptor, HBM memory map, validation,
// split planning, launches and the canonical export.
//
// Everything is validated on the host before a launch; a failing call launches nothing
// and leaves the cache length unchanged. No device memory is allocated here.
#include "../../include/kvq.h"
#include "kvq_internal.cuh"

#include <cstring>
#include <new>
#include <vector>

using namespace kvq;

struct kvq_cache {
    kvq_layout L;
    int kf, vf, tf, W;
    RowFmt fmt[2], tail;
    // byte offsets of the areas inside the bound buffer
    size_t off_main[2], off_ring[2], off_scales, off_pend, off_meta;
    size_t main_region[2], ring_region;   // bytes per (layer, b, h) region
    size_t total;
    uint8_t* buf;
    size_t buf_bytes;
    int device, num_sms;
    std::vector<long long> n;            // per layer
    std::vector<char> scales_set;        // per layer (kvarn)
};

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// metadata region: a 256-byte header (word 0 = device status) and 4 uint32 value bounds per
// (layer, batch element, kv head)
constexpr size_t META_HEADER_WORDS = 64;
size_t meta_bytes(const kvq_layout& L) {
    return align_up(META_HEADER_WORDS * 4 + (size_t)L.n_layers * L.batch * L.n_kv_heads * 4 * sizeof(uint32_t), 256);
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

LayerView layer_view(const kvq_cache* c, int layer) {
    LayerView v{};
    const size_t units = (size_t)c->L.batch * c->L.n_kv_heads;
    for (int kv = 0; kv < 2; ++kv) {
        v.main[kv] = c->buf + c->off_main[kv] + (size_t)layer * units * c->main_region[kv];
        v.ring[kv] = c->W ? c->buf + c->off_ring[kv] + (size_t)layer * units * c->ring_region : nullptr;
        v.fmt[kv] = c->fmt[kv];
    }
    v.main_region[0] = (long long)c->main_region[0];
    v.main_region[1] = (long long)c->main_region[1];
    v.ring_region = (long long)c->ring_region;
    v.scales = c->L.kvarn ? reinterpret_cast<float*>(c->buf + c->off_scales) +
                                (size_t)layer * units * 2 * c->L.head_dim
                          : nullptr;
    v.tail = c->tail;
    uint32_t* meta = reinterpret_cast<uint32_t*>(c->buf + c->off_meta);
    v.kivi = c->L.k_per_channel;
    v.kbb = block_bytes(c->kf);
    v.pend = c->L.k_per_channel ? reinterpret_cast<float*>(c->buf + c->off_pend) + (size_t)layer * units * 32 * c->L.head_dim
                                : nullptr;
    v.status = meta;
    v.stats = meta + META_HEADER_WORDS + (size_t)layer * units * 4;
    v.B = c->L.batch;
    v.H = c->L.n_kv_heads;
    v.D = c->L.head_dim;
    v.G = c->L.n_q_heads / c->L.n_kv_heads;
    v.W = c->W;
    v.kvarn = c->L.kvarn;
    return v;
}

kvq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

// device address of the no-allocation workspace on `dev` (defined with the entry point below)
kvq_status noalloc_workspace(int dev, void** ptr);

}  // namespace

extern "C" {

const char* kvq_status_string(kvq_status s) {
    switch (s) {
        case KVQ_OK: return "ok";
        case KVQ_ERR_INVALID_ARG: return "invalid argument";
        case KVQ_ERR_UNSUPPORTED_FMT: return "unsupported format";
        case KVQ_ERR_CAPACITY: return "capacity exceeded";
        case KVQ_ERR_CALIBRATION: return "KVarN calibration needs a longer first append";
        case KVQ_ERR_EMPTY: return "empty cache";
        case KVQ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case KVQ_ERR_NOT_BOUND: return "no device buffer bound";
        case KVQ_ERR_CUDA: return "CUDA error";
        case KVQ_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait on the device ran out";
    }
    return "unknown status";
}

kvq_status kvq_cache_create(const kvq_layout* layout, kvq_fmt k_fmt, kvq_fmt v_fmt, kvq_fmt tail_fmt,
                            int32_t W, kvq_cache** out) {
    if (!layout || !out) return KVQ_ERR_INVALID_ARG;
    *out = nullptr;
    const kvq_layout& L = *layout;
    if (L.n_layers < 1 || L.batch < 1 || L.n_kv_heads < 1 || L.n_q_heads < L.n_kv_heads ||
        L.n_q_heads % L.n_kv_heads || L.max_ctx < 1 || L.max_ctx > (1LL << 31))
        return KVQ_ERR_INVALID_ARG;
    if (L.k_per_channel != 0 && L.k_per_channel != 1) return KVQ_ERR_INVALID_ARG;
    if (L.k_per_channel && L.kvarn) return KVQ_ERR_INVALID_ARG;
    const int D = L.head_dim;
    if (D != 32 && D != 64 && D != 128 && D != 256) return KVQ_ERR_INVALID_ARG;
    const int G = L.n_q_heads / L.n_kv_heads;
    if (G > 8) return KVQ_ERR_INVALID_ARG;
    if (L.kvarn != 0 && L.kvarn != 1) return KVQ_ERR_INVALID_ARG;
    if (L.kvarn) {
        const int T = L.kvarn_calib_tokens;
        if (T < 64 || T > 1024 || (T & (T - 1)) || !(L.kvarn_eps >= 0.0)) return KVQ_ERR_INVALID_ARG;
    }
    if (!is_lowbit(k_fmt) || !is_lowbit(v_fmt)) return KVQ_ERR_UNSUPPORTED_FMT;
    if (W < 0 || W > L.max_ctx) return KVQ_ERR_INVALID_ARG;
    if (W == 0 && tail_fmt != KVQ_NONE) return KVQ_ERR_INVALID_ARG;
    if (W > 0 && !(tail_fmt == KVQ_Q8_0 || tail_fmt == KVQ_BF16 || tail_fmt == KVQ_F16))
        return KVQ_ERR_UNSUPPORTED_FMT;

    kvq_cache* c = new (std::nothrow) kvq_cache();
    if (!c) return KVQ_ERR_INVALID_ARG;
    c->L = L;
    c->kf = k_fmt; c->vf = v_fmt; c->tf = tail_fmt; c->W = W;
    c->fmt[0] = make_rowfmt(k_fmt, D);
    c->fmt[1] = make_rowfmt(v_fmt, D);
    if (W) c->tail = make_rowfmt(tail_fmt, D);
    const size_t units = (size_t)L.n_layers * L.batch * L.n_kv_heads;
    size_t off = 0;
    for (int kv = 0; kv < 2; ++kv) {
        c->main_region[kv] = align_up((size_t)L.max_ctx * c->fmt[kv].stride, 256);
        if (kv == 0 && L.k_per_channel)   // whole groups of 32 positions of D blocks
            c->main_region[kv] = align_up((size_t)((L.max_ctx + 31) / 32) * D * block_bytes(k_fmt), 256);
        c->off_main[kv] = off;
        off += units * c->main_region[kv];
    }
    c->ring_region = W ? align_up((size_t)W * c->tail.stride, 256) : 0;
    for (int kv = 0; kv < 2; ++kv) {
        c->off_ring[kv] = off;
        off += units * c->ring_region;
    }
    c->off_scales = off;
    if (L.kvarn) off += align_up(units * 2 * D * sizeof(float), 256);
    c->off_pend = off;
    if (L.k_per_channel) off += align_up(units * 32 * D * sizeof(float), 256);
    c->off_meta = off;
    off += meta_bytes(L);
    c->total = off;
    c->buf = nullptr;
    c->buf_bytes = 0;
    c->device = -1;
    c->num_sms = 0;
    c->n.assign(L.n_layers, 0);
    c->scales_set.assign(L.n_layers, 0);
    *out = c;
    return KVQ_OK;
}

kvq_status kvq_cache_required_bytes(const kvq_cache* c, size_t* bytes) {
    if (!c || !bytes) return KVQ_ERR_INVALID_ARG;
    *bytes = c->total;
    return KVQ_OK;
}

kvq_status kvq_cache_bind(kvq_cache* c, void* dev_buf, size_t bytes, void* stream) {
    if (!c || !dev_buf) return KVQ_ERR_INVALID_ARG;
    if (((uintptr_t)dev_buf & 255) != 0) return KVQ_ERR_ALIGNMENT;
    if (bytes < c->total) return KVQ_ERR_CAPACITY;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return KVQ_ERR_CUDA;
    if (cudaMemsetAsync(dev_buf, 0, c->total, (cudaStream_t)stream) != cudaSuccess) return KVQ_ERR_CUDA;
    // map the no-allocation entry point's fixed array now, while the caller is setting up,
    // rather than at its first call (lazy module loading maps it at the first lookup)
    void* ws = nullptr;
    kvq_status s = noalloc_workspace(dev, &ws);
    if (s != KVQ_OK) return s;
    c->buf = (uint8_t*)dev_buf;
    c->buf_bytes = bytes;
    c->device = dev;
    c->num_sms = sms;
    std::fill(c->n.begin(), c->n.end(), 0);
    std::fill(c->scales_set.begin(), c->scales_set.end(), 0);
    return KVQ_OK;
}

kvq_status kvq_cache_destroy(kvq_cache* c) {
    delete c;
    return KVQ_OK;
}

kvq_status kvq_length(const kvq_cache* c, int32_t layer, int64_t* n) {
    if (!c || !n || layer < 0 || layer >= c->L.n_layers) return KVQ_ERR_INVALID_ARG;
    *n = c->n[layer];
    return KVQ_OK;
}

kvq_status kvq_set_channel_scales(kvq_cache* c, int32_t layer, const float* sK, const float* sV, void* stream) {
    if (!c || !sK || !sV || layer < 0 || layer >= c->L.n_layers || !c->L.kvarn) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    if (!aligned16(sK) || !aligned16(sV)) return KVQ_ERR_ALIGNMENT;
    if (c->n[layer] != 0) return KVQ_ERR_INVALID_ARG;
    const LayerView v = layer_view(c, layer);
    const size_t row = (size_t)c->L.head_dim * sizeof(float);
    // device layout [B][H][2][D]: interleave K and V rows with two strided copies
    const int BH = c->L.batch * c->L.n_kv_heads;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpy2DAsync(v.scales, 2 * row, sK, row, row, BH, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpy2DAsync((uint8_t*)v.scales + row, 2 * row, sV, row, row, BH, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return KVQ_ERR_CUDA;
    c->scales_set[layer] = 1;
    return KVQ_OK;
}

kvq_status kvq_get_channel_scales(const kvq_cache* c, int32_t layer, float* host_sK, float* host_sV) {
    if (!c || !host_sK || !host_sV || layer < 0 || layer >= c->L.n_layers || !c->L.kvarn) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    if (!c->scales_set[layer]) return KVQ_ERR_CALIBRATION;
    const LayerView v = layer_view(c, layer);
    const size_t row = (size_t)c->L.head_dim * sizeof(float);
    const int BH = c->L.batch * c->L.n_kv_heads;
    if (cudaDeviceSynchronize() != cudaSuccess) return KVQ_ERR_CUDA;
    if (cudaMemcpy2D(host_sK, row, v.scales, 2 * row, row, BH, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy2D(host_sV, row, (const uint8_t*)v.scales + row, 2 * row, row, BH, cudaMemcpyDeviceToHost) != cudaSuccess)
        return KVQ_ERR_CUDA;
    return KVQ_OK;
}

kvq_status kvq_device_status(kvq_cache* c, void* stream) {
    if (!c) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t* word = reinterpret_cast<uint32_t*>(c->buf + c->off_meta);
    uint32_t h = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return KVQ_ERR_CUDA;
    if (cudaMemcpy(&h, word, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return KVQ_ERR_CUDA;
    if (h == 0) return KVQ_OK;
    if (cudaMemsetAsync(word, 0, sizeof(uint32_t), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
        return KVQ_ERR_CUDA;
    return KVQ_ERR_DEVICE_TIMEOUT;
}

kvq_status kvq_selftest_wait_timeout(kvq_cache* c, uint64_t limit_ns, void* stream) {
    if (!c || limit_ns > 10000000000ull) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    uint32_t* word = reinterpret_cast<uint32_t*>(c->buf + c->off_meta);
    return cuda_status(launch_wait_selftest(word, (unsigned long long)limit_ns, (cudaStream_t)stream));
}

kvq_status kvq_append(kvq_cache* c, int32_t layer, const float* k, const float* v, int32_t n_new, void* stream) {
    if (!c || layer < 0 || layer >= c->L.n_layers || n_new < 0) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    if (n_new == 0) return KVQ_OK;
    if (!k || !v) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v)) return KVQ_ERR_ALIGNMENT;
    const long long n = c->n[layer];
    if (n + n_new > c->L.max_ctx) return KVQ_ERR_CAPACITY;
    cudaStream_t st = (cudaStream_t)stream;
    const LayerView lv = layer_view(c, layer);
    if (c->L.kvarn && !c->scales_set[layer]) {
        if (n != 0 || n_new < c->L.kvarn_calib_tokens) return KVQ_ERR_CALIBRATION;
        kvq_status s = cuda_status(launch_calibrate(lv, k, v, n_new, c->L.kvarn_calib_tokens, c->L.kvarn_eps, st));
        if (s != KVQ_OK) return s;
        c->scales_set[layer] = 1;
    }
    kvq_status s = cuda_status(launch_append(lv, k, v, n, n_new, st));
    if (s != KVQ_OK) return s;
    c->n[layer] = n + n_new;
    return KVQ_OK;
}

kvq_status kvq_decode_workspace_bytes(const kvq_cache* c, int32_t n_query_rows, size_t* bytes) {
    if (!c || !bytes || n_query_rows < 1) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    const long long units = (long long)c->L.batch * c->L.n_kv_heads * n_query_rows;
    // main and ring splits are each at most per_unit + 1 (see plan_splits)
    const long long per_unit = (4LL * c->num_sms + units - 1) / units;
    const long long max_split = 2 * (per_unit < 1 ? 1 : per_unit) + 2;
    const int G = c->L.n_q_heads / c->L.n_kv_heads;
    *bytes = (size_t)units * max_split * partial_floats(G, c->L.head_dim) * sizeof(float);
    // a tensor-core prefill keeps its key-range partials here, after the dequantized tile
    // images on the staged path
    if (!c->L.k_per_channel && prefill_supported(c->L.head_dim) && n_query_rows > 1) {
        const size_t img = prefill_staged_used(c->L.head_dim, n_query_rows, G)
                               ? align_up(prefill_image_bytes(c->L.batch, c->L.n_kv_heads, c->L.head_dim, c->L.max_ctx), 256)
                               : 0;
        const size_t all = img + prefill_partial_bytes(c->L.batch, c->L.n_kv_heads, c->L.n_q_heads, c->L.head_dim,
                                                       n_query_rows);
        if (all > *bytes) *bytes = all;
    }
    return KVQ_OK;
}

static kvq_status attention_common(kvq_cache* c, int32_t layer, const float* q, int rows, float scale,
                                   float* out, void* ws, size_t ws_bytes, void* stream) {
    if (!c || layer < 0 || layer >= c->L.n_layers || !q || !out || !ws) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    if (!aligned16(q) || !aligned16(out) || !aligned16(ws)) return KVQ_ERR_ALIGNMENT;
    const long long n = c->n[layer];
    if (n == 0) return KVQ_ERR_EMPTY;
    if (rows < 1 || rows > n) return KVQ_ERR_INVALID_ARG;
    size_t need = 0;
    kvq_status s = kvq_decode_workspace_bytes(c, rows, &need);
    if (s != KVQ_OK) return s;
    if (ws_bytes < need) return KVQ_ERR_CAPACITY;
    const LayerView lv = layer_view(c, layer);
    const long long n_ring = c->W ? (n < c->W ? n : c->W) : 0;
    const long long units = (long long)c->L.batch * c->L.n_kv_heads * rows;
    const int tc_ctas = (use_tensor_cores(c->L.head_dim) && !c->L.k_per_channel) ? tc_ctas_per_sm(c->L.head_dim) : 0;
    const SplitPlan plan = plan_splits(n - n_ring, n_ring, units, c->num_sms, tc_ctas);
    return cuda_status(launch_attention(lv, q, scale, out, (float*)ws, n, rows, plan, (cudaStream_t)stream));
}

kvq_status kvq_decode_attention(kvq_cache* c, int32_t layer, const float* q, float scale, float* out, void* ws,
                                size_t ws_bytes, void* stream) {
    return attention_common(c, layer, q, 1, scale, out, ws, ws_bytes, stream);
}

kvq_status kvq_decode_attention_indexed(kvq_cache* c, int32_t layer, const float* q, float scale,
                                        const int32_t* idx, int32_t n_idx, float* out, void* ws, size_t ws_bytes,
                                        void* stream) {
    if (!c || layer < 0 || layer >= c->L.n_layers || !q || !out || !ws || !idx) return KVQ_ERR_INVALID_ARG;
    if (n_idx < 1 || n_idx > KVQ_MAX_GATHER) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    if (!aligned16(q) || !aligned16(out) || !aligned16(ws) || ((uintptr_t)idx & 3)) return KVQ_ERR_ALIGNMENT;
    const long long n = c->n[layer];
    if (n == 0) return KVQ_ERR_EMPTY;
    size_t need = 0;
    kvq_status s = kvq_decode_workspace_bytes(c, 1, &need);
    if (s != KVQ_OK) return s;
    if (ws_bytes < need) return KVQ_ERR_CAPACITY;
    const LayerView lv = layer_view(c, layer);
    // both passes walk the whole list; a pass whose region holds no position is skipped
    const long long list_main = (c->W == 0 || n > c->W) ? n_idx : 0;
    const long long list_ring = c->W ? n_idx : 0;
    const long long units = (long long)c->L.batch * c->L.n_kv_heads;
    const int tc_ctas = (use_tensor_cores(c->L.head_dim) && !c->L.k_per_channel) ? tc_ctas_per_sm(c->L.head_dim) : 0;
    const SplitPlan plan = plan_splits(list_main, list_ring, units, c->num_sms, tc_ctas);
    return cuda_status(launch_attention(lv, q, scale, out, (float*)ws, n, 1, plan, (cudaStream_t)stream, idx, n_idx));
}

kvq_status kvq_prefill_attention(kvq_cache* c, int32_t layer, const float* q, int32_t n_chunk, float scale,
                                 float* out, void* ws, size_t ws_bytes, void* stream) {
    if (n_chunk < 1) return KVQ_ERR_INVALID_ARG;
    // Chunks of up to 4 rows (a multi-query verify) take the split-K decode kernel, one pass
    // over the keys per row, which streams the cache at the decode's rate; longer chunks take
    // the tcgen05 prefill, whose cost does not grow with the rows of an M-tile.
    constexpr int DECODE_PATH_ROWS = 4;
    if (c && prefill_supported(c->L.head_dim) && !c->L.k_per_channel && n_chunk > DECODE_PATH_ROWS) {
        // tensor-core path: validated like the split-K path, needs no workspace
        if (layer < 0 || layer >= c->L.n_layers || !q || !out || !ws) return KVQ_ERR_INVALID_ARG;
        if (!c->buf) return KVQ_ERR_NOT_BOUND;
        if (!aligned16(q) || !aligned16(out) || !aligned16(ws)) return KVQ_ERR_ALIGNMENT;
        const long long n = c->n[layer];
        if (n == 0) return KVQ_ERR_EMPTY;
        if (n_chunk > n) return KVQ_ERR_INVALID_ARG;
        size_t need = 0;
        kvq_status s = kvq_decode_workspace_bytes(c, n_chunk, &need);
        if (s != KVQ_OK) return s;
        if (ws_bytes < need) return KVQ_ERR_CAPACITY;
        const int G = c->L.n_q_heads / c->L.n_kv_heads;
        const bool staged = prefill_staged_used(c->L.head_dim, n_chunk, G);
        // the key-range partials follow the tile images (staged path) or fill the workspace
        const size_t img = staged ? align_up(prefill_image_bytes(c->L.batch, c->L.n_kv_heads, c->L.head_dim,
                                                                 c->L.max_ctx), 256)
                                  : 0;
        return cuda_status(launch_prefill(layer_view(c, layer), q, scale, out, n, n_chunk, (cudaStream_t)stream,
                                          staged ? (uint8_t*)ws : nullptr, staged ? (c->L.max_ctx + 31) / 32 : 0,
                                          (float*)((uint8_t*)ws + img), ws_bytes - img, c->num_sms));
    }
    return attention_common(c, layer, q, n_chunk, scale, out, ws, ws_bytes, stream);
}

kvq_status kvq_export_blocks(const kvq_cache* c, int32_t layer, int32_t b, int32_t h, int32_t kv, int32_t region,
                             int64_t pos0, int64_t count, void* host_dst, size_t bytes) {
    if (!c || !host_dst || layer < 0 || layer >= c->L.n_layers || b < 0 || b >= c->L.batch || h < 0 ||
        h >= c->L.n_kv_heads || kv < 0 || kv > 1 || pos0 < 0 || count < 0)
        return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    const RowFmt* f;
    const uint8_t* base;
    const LayerView lv = layer_view(c, layer);
    const int D = c->L.head_dim, nb = D / 32;
    if (kv == 0 && c->L.k_per_channel && (region == 0 || region == 2)) {
        // per-channel K: region 0 = groups pos0.. (D canonical blocks each, stored as is),
        // region 2 = pending slots pos0.. (float32 rows)
        const size_t unit = (size_t)(b * c->L.n_kv_heads + h);
        size_t per, lim;
        const uint8_t* src;
        if (region == 0) {
            per = (size_t)D * block_bytes(c->kf);
            lim = (size_t)((c->L.max_ctx + 31) / 32);
            src = lv.main[0] + unit * c->main_region[0];
        } else {
            per = (size_t)D * sizeof(float);
            lim = 32;
            src = reinterpret_cast<const uint8_t*>(lv.pend + unit * 32 * D);
        }
        if ((size_t)(pos0 + count) > lim) return KVQ_ERR_INVALID_ARG;
        if (bytes < (size_t)count * per) return KVQ_ERR_CAPACITY;
        if (count == 0) return KVQ_OK;
        if (cudaDeviceSynchronize() != cudaSuccess) return KVQ_ERR_CUDA;
        if (cudaMemcpy(host_dst, src + (size_t)pos0 * per, (size_t)count * per, cudaMemcpyDeviceToHost) != cudaSuccess)
            return KVQ_ERR_CUDA;
        return KVQ_OK;
    }
    if (region == 0) {
        if (pos0 + count > c->L.max_ctx) return KVQ_ERR_INVALID_ARG;
        f = &c->fmt[kv];
        base = lv.main[kv] + (size_t)(b * c->L.n_kv_heads + h) * c->main_region[kv];
    } else if (region == 1) {
        if (!c->W || pos0 + count > c->W) return KVQ_ERR_INVALID_ARG;
        f = &c->tail;
        base = lv.ring[kv] + (size_t)(b * c->L.n_kv_heads + h) * c->ring_region;
    } else {
        return KVQ_ERR_INVALID_ARG;
    }
    const size_t canon_row = (size_t)f->row_bytes;   // same bytes, block-major order
    if (bytes < (size_t)count * canon_row) return KVQ_ERR_CAPACITY;
    if (count == 0) return KVQ_OK;
    std::vector<uint8_t> tmp((size_t)count * f->stride);
    if (cudaDeviceSynchronize() != cudaSuccess) return KVQ_ERR_CUDA;
    if (cudaMemcpy(tmp.data(), base + (size_t)pos0 * f->stride, tmp.size(), cudaMemcpyDeviceToHost) != cudaSuccess)
        return KVQ_ERR_CUDA;
    uint8_t* dst = (uint8_t*)host_dst;
    for (int64_t r = 0; r < count; ++r) {
        const uint8_t* row = tmp.data() + (size_t)r * f->stride;
        uint8_t* o = dst + (size_t)r * canon_row;
        if (f->kind != 0) {
            std::memcpy(o, row, canon_row);
            continue;
        }
        for (int blk = 0; blk < nb; ++blk) {
            std::memcpy(o, row + 2 * blk, 2); o += 2;
            if (f->asym) { std::memcpy(o, row + f->off_m + 2 * blk, 2); o += 2; }
            // a block's plane bytes are its four 8-channel pieces in order
            for (int t = 0; t < 4; ++t) { std::memcpy(o, row + f->off_p0 + piece_off(nb, blk, t, f->w0), f->w0); o += f->w0; }
            if (f->w1)
                for (int t = 0; t < 4; ++t) { std::memcpy(o, row + f->off_p1 + piece_off(nb, blk, t, f->w1), f->w1); o += f->w1; }
        }
    }
    return KVQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without any device allocation.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: for example a
// plugin running inside a host program that owns the device allocator and gives its
// extensions no way to reach it, or a C caller that must keep its device footprint fixed
// once it has started. kvq_decode_attention_noalloc serves them by running the same
// split-K decode with its softmax partials in the fixed array below instead of a
// caller-provided workspace.
//
// The array lives in this library's device image: every GPU on which the library is
// loaded holds its KVQ_NOALLOC_WS_BYTES until the process exits. In host code its name
// only stands for the device symbol; the device address is looked up once per device
// with cudaGetSymbolAddress (when a cache is first bound on that device, or at the entry
// point's first call there, with that device current) and cached. Every call shares the array and it keeps the last call's
// contents; the decode's first pass writes every partial the merge reads, so nothing has
// to start at zero. Calls whose kernels overlap on the GPU (several streams, several
// threads) race on the array.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {
constexpr size_t KVQ_NOALLOC_WS_BYTES = (size_t)KVQ_NOALLOC_WORKSPACE_MIB << 20;
constexpr int KVQ_MAX_DEVICES = 64;
static __device__ __align__(256) unsigned char g_noalloc_ws[KVQ_NOALLOC_WS_BYTES];
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[KVQ_MAX_DEVICES] = {};

// Device address of g_noalloc_ws on `dev` (which must be current), looked up once.
kvq_status noalloc_workspace(int dev, void** ptr) {
    if (dev < 0 || dev >= KVQ_MAX_DEVICES) return KVQ_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) return KVQ_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return KVQ_OK;
}
}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(kvq_cache* c, int32_t layer, const float* q, float scale,
                                                   float* out, void* stream) {
    if (!c || layer < 0 || layer >= c->L.n_layers || !q || !out) return KVQ_ERR_INVALID_ARG;
    if (!c->buf) return KVQ_ERR_NOT_BOUND;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
    if (dev != c->device) return KVQ_ERR_INVALID_ARG;
    size_t need = 0;
    kvq_status s = kvq_decode_workspace_bytes(c, 1, &need);
    if (s != KVQ_OK) return s;
    if (need > KVQ_NOALLOC_WS_BYTES) return KVQ_ERR_CAPACITY;
    void* ws = nullptr;
    s = noalloc_workspace(dev, &ws);
    if (s != KVQ_OK) return s;
    return attention_common(c, layer, q, 1, scale, out, ws, KVQ_NOALLOC_WS_BYTES, stream);
}
