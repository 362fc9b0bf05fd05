// kvq_internal.cuh -- device-side layout, format descriptors and kernel entry points
// shared by the libkvq translation units (CUDA path only).
//
// HBM layout of a bound cache (all regions 256-byte aligned):
//   K main  [L][B][H] regions of max_ctx rows (K format row stride)
//   V main  [L][B][H] regions of max_ctx rows (V format row stride)
//   K ring  [L][B][H] regions of W rows (tail format row stride)        (W > 0)
//   V ring  [L][B][H] regions of W rows                                  (W > 0)
//   scales  [L][B][H][2][D] float32 KVarN channel scales                 (kvarn)
//   pending [L][B][H] 32 x D float32 rows                                 (per-channel K)
//   meta    256-byte header (word 0: device status, bits set by a kernel whose bounded
//           wait ran out) then stats [L][B][H][2 (K|V)][2] uint32: float bits of upper
//           bounds of |value| over every row stored so far, [0] in the stored domain
//           (the block values d*c (+m), before the KVarN channel scale) and [1] in the
//           dequantized domain (after it). Kernels use them to pick power-of-two scalings
//           that keep 16-bit tensor-core operands inside the fp16 range.
// A low-bit row of D channels (nb = D/32 blocks) is stored as
//   [d: nb x fp16][m: nb x fp16, qX_1 only][plane0: D*w0/8 bytes][plane1: D*w1/8 bytes]
// padded to 16 bytes. A plane holds the X-bit codes' low w0 bits (plane 0) or next w1 bits
// (plane 1) in pieces of 8 channels: piece (b, t) = channels 32b + 8t .. 32b + 8t + 7 of
// block b, t = 0..3, is the little-endian bitstream of those 8 codes (channel 32b + 8t + j at
// bits [j*w, j*w + w)), w bytes long, stored at byte (t * nb + b) * w of the plane. Slot t of
// consecutive blocks is contiguous, so a thread that handles slot t of several blocks reads
// them with one wide load. The canonical per-block serialisation is a byte permutation of
// this row (block b of a plane = its pieces t = 0..3 in order). A bf16 / f16 row is D x 2
// bytes in channel order.
// With per-channel K (token-axis blocks), the K main area of a (layer, b, h) instead holds
// groups of 32 positions, each group D canonical blocks in channel order (block (g, c) at
// byte (g * D + c) * block_bytes: d | [m] | plane0 | plane1, code t of the block = position
// 32 g + t at bits [t*w, t*w + w) of each plane); positions that entered the K store but
// whose group is not complete are float32 rows in the pending area, slot pos mod 32.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace kvq {

enum : int {
    F_Q2_0 = 0, F_Q2_1, F_Q3_0, F_Q3_1, F_Q4_0, F_Q4_1, F_Q5_0, F_Q5_1, F_Q6_0, F_Q6_1, F_Q8_0, F_Q8_1,
    F_BF16 = 12, F_F16 = 13, F_NONE = 14
};

__host__ __device__ inline bool is_lowbit(int f) { return f >= F_Q2_0 && f <= F_Q8_1; }
__host__ __device__ inline int fmt_bits(int f) {
    return is_lowbit(f) ? ((f / 2 == 5) ? 8 : 2 + f / 2) : 16;
}
__host__ __device__ inline bool fmt_asym(int f) { return is_lowbit(f) && (f & 1); }

// Runtime description of one row format (same for main-store and ring rows).
struct RowFmt {
    int id;        // kvq_fmt value
    int kind;      // 0: block-quantized, 1: bf16, 2: f16
    int bits;      // X
    int asym;      // qX_1
    int w0, w1;    // plane widths, low bits first (w1 = 0: one plane)
    int off_m;     // byte offset of the mins
    int off_p0;    // byte offset of plane 0
    int off_p1;    // byte offset of plane 1
    int stride;    // row stride in bytes (multiple of 16)
    int row_bytes; // unpadded bytes of one row
};

// Byte offset, inside a plane of w-bit codes of a row with nb blocks, of the 8-channel
// piece (b, t) (see the layout above).
__host__ __device__ constexpr int piece_off(int nb, int b, int t, int w) { return (t * nb + b) * w; }
// Bit offset, inside such a plane, of channel c's code.
__host__ __device__ constexpr int plane_bit(int nb, int c, int w) {
    return piece_off(nb, c >> 5, (c >> 3) & 3, w) * 8 + (c & 7) * w;
}

__host__ inline RowFmt make_rowfmt(int f, int D) {
    RowFmt r{};
    r.id = f;
    const int nb = D / 32;
    if (f == F_BF16 || f == F_F16) {
        r.kind = (f == F_BF16) ? 1 : 2;
        r.bits = 16;
        r.row_bytes = 2 * D;
    } else {
        r.kind = 0;
        r.bits = fmt_bits(f);
        r.asym = fmt_asym(f) ? 1 : 0;
        switch (r.bits) {
            case 8: r.w0 = 8; r.w1 = 0; break;
            case 6: r.w0 = 4; r.w1 = 2; break;
            case 5: r.w0 = 4; r.w1 = 1; break;
            case 4: r.w0 = 4; r.w1 = 0; break;
            case 3: r.w0 = 2; r.w1 = 1; break;
            default: r.w0 = 2; r.w1 = 0; break;
        }
        r.off_m = 2 * nb;
        r.off_p0 = 2 * nb * (r.asym ? 2 : 1);
        r.off_p1 = r.off_p0 + D * r.w0 / 8;
        r.row_bytes = r.off_p1 + D * r.w1 / 8;
    }
    r.stride = (r.row_bytes + 15) & ~15;
    return r;
}

// Per-layer view handed to kernels.
struct LayerView {
    uint8_t* main[2];      // K / V main area of this layer: [B][H] regions
    uint8_t* ring[2];      // K / V ring area of this layer (nullptr if W == 0)
    float* scales;         // [B][H][2][D] (nullptr unless kvarn)
    long long main_region[2]; // K / V bytes per (b, h) main region
    long long ring_region; // bytes per (b, h) ring region
    RowFmt fmt[2];         // K / V low-bit formats
    RowFmt tail;           // tail format (kind 0 = q8_0)
    uint32_t* stats;       // this layer's [B][H][2][2] value bounds (see the layout above)
    float* pend;           // per-channel K: this layer's [B][H] pending rows (else nullptr)
    int kivi;              // per-channel (token-axis) K blocks
    int kbb;               // per-channel K: canonical block bytes of the K format
    uint32_t* status;      // the cache's device status word
    int B, H, D, G, W;
    int kvarn;
};

// device status bits
constexpr uint32_t STATUS_WAIT_TIMEOUT = 1u;

// Power-of-two exponent e such that bound * 2^-e < 2^15 with bound * 2^-e >= 2^14 (0 for a
// zero or non-finite bound), clamped to [lo, hi].
__host__ __device__ inline int pow2_exponent(float bound, int lo, int hi) {
    if (!(bound > 0.f) || !(bound < 3.0e38f)) return 0;
    int e = 0;
    (void)frexpf(bound, &e);       // bound = f * 2^e, f in [0.5, 1)
    e -= 15;
    return e < lo ? lo : (e > hi ? hi : e);
}

// Scaling for 16-bit tensor-core operands: a value range whose maximum m already lies in
// [2^-4, 2^14) is left alone (exponent 0); otherwise m * 2^-e lands in [2^14, 2^15), inside
// fp16's range with the normal-range precision of its hi + lo split for all but values
// 2^18 times smaller than m.
__host__ __device__ inline int fp16_exponent(float m, int lo, int hi) {
    if (m >= 0.0625f && m < 16384.f) return 0;
    return pow2_exponent(m, lo, hi);
}

// ---------------------------------------------------------------- launches
cudaError_t launch_append(const LayerView& lv, const float* k, const float* v, long long n, int C,
                          cudaStream_t st);
// block bytes of a format (2 + 4X, or 4 + 4X for qX_1)
__host__ __device__ inline int block_bytes(int f) { return (fmt_asym(f) ? 4 : 2) + 4 * fmt_bits(f); }
cudaError_t launch_calibrate(const LayerView& lv, const float* k, const float* v, int C, int T,
                             double eps, cudaStream_t st);

// Split plan of one attention call: every (b, h, query row) unit is cut into
// n_main_split pieces over the low-bit rows and n_ring_split pieces over the ring.
struct SplitPlan {
    int n_main_split, n_ring_split;
    long long main_chunk, ring_chunk;  // rows per split
    int n_split() const { return n_main_split + n_ring_split; }
};
// Tensor-core path (head_dim 128 / 256) when tc is set: splits are whole 64-row tiles.
// tc_ctas: CTAs per SM of the tensor-core decode kernel (0: CUDA-core path)
SplitPlan plan_splits(long long n_main, long long n_ring, long long units, int num_sms, int tc_ctas);
int tc_ctas_per_sm(int head_dim);
bool use_tensor_cores(int D);
size_t partial_floats(int G, int D);   // floats of one split partial

// rows = query rows per (b, h): 1 for decode, n_chunk for prefill. q/out layout
// [B][rows][Hq][D]. pos_base: position of query row 0 (n - rows); decode uses rows = 1
// and pos_base = n - 1 so every row sees all n positions.
// idx (optional): index-gather decode (rows = 1), [B][H][n_idx] positions per (b, h); the
// low-bit and ring passes then both run over the list entries.
cudaError_t launch_attention(const LayerView& lv, const float* q, float scale, float* out,
                             float* ws, long long n, int rows, const SplitPlan& plan,
                             cudaStream_t st, const int* idx = nullptr, int n_idx = 0);

// Chunked prefill on tcgen05 (head_dim 128 / 256): q, out [B][C][Hq][D], n = cached
// positions after the chunk's append.
bool prefill_supported(int D);
// The staged prefill (tiles dequantized once per (b, h) into a workspace image area, then
// streamed by every M-tile CTA) runs when a head has more than one 128-row M-tile.
bool prefill_staged_used(int D, int C, int G);
size_t prefill_image_bytes(int B, int H, int D, long long max_ctx);
// partials of a tensor-core prefill whose M-tiles are split over the key range (H kv heads,
// Hq query heads, a chunk of C rows)
size_t prefill_partial_bytes(int B, int H, int Hq, int D, int C);
// img: image area of prefill_image_bytes(B, H, D, img_tiles * 32) bytes for the staged
// kernel, or nullptr for the on-the-fly kernel; part: prefill_partial_bytes of workspace
// (nullptr: no key-range splits) of part_bytes (caps the split count), num_sms: the device's
// SM count (picks the split count)
cudaError_t launch_prefill(const LayerView& lv, const float* q, float scale, float* out, long long n, int C,
                           cudaStream_t st, uint8_t* img = nullptr, long long img_tiles = 0,
                           float* part = nullptr, size_t part_bytes = 0, int num_sms = 0);

// One warp waits, with the bounded wait the pipelined kernels use and a limit of limit_ns,
// on an mbarrier that nothing ever arrives on, then records the timeout in *status.
cudaError_t launch_wait_selftest(uint32_t* status, unsigned long long limit_ns, cudaStream_t st);

}  // namespace kvq
