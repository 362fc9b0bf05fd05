/*
 * kvq_oracle.cpp -- plain scalar CPU oracle for attention over a block-quantized,
 * mixed-precision KV cache.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg load this library. It shares no code, header,
 * table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * Build: g++ -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (no FMA contraction,
 * IEEE float division, correctly rounded sqrt/exp from the C library).
 *
 * Sources (web pages; cited by title and section):
 *   [KVBENCH]  "KV cache quant benchmarks: KVarN 6-bit matches q8_0, 4-bit matches q5_0"
 *              -- cache-size table (bf16 / q8_0 / q6_0 / q5_1 / pair rows).
 *   [HARDNUM]  "Hard numbers on Qwen3.8-27B's KV cache: q8_0 is free, K is ~2x as touchy
 *              as V, and a 2k recent-token window makes 6/5-bit basically lossless"
 *              -- sections "KV cache low-bit storage" and "Reddit reactions".
 *   [BEELLAMA] "BeeLlama.cpp v0.4.1: KVarN, KV precision tail, q2_0-q3_1 KV cache"
 *              -- "KV cache precision tail" paragraph, new-types paragraph, KV-MiB table.
 *   [OFFLOAD]  "You can offload most of Qwen3.8-Flash-Next's KV cache to RAM with little
 *              decode slowdown" -- row-size arithmetic paragraph.
 *
 * The pages print no formulas. Where they are silent the oracle takes the plainest
 * reading; each such reading is marked READING below.
 *
 * Parity pins: every function here is pinned by a test that does not re-type its
 * formula (closed-form byte counts, exhaustive conversion checks against host
 * hardware, brute-force code search, attention special cases, an independent
 * library attention routine). See the tests' docstrings for which pin covers what.
 */
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

// ---------------------------------------------------------------------------
// Formats. Enum values mirror the public C ABI's kvq_fmt order (an interface
// that must match; the numbers are the ABI contract, the code is separate).
// ---------------------------------------------------------------------------
enum Fmt {
    Q2_0 = 0, Q2_1, Q3_0, Q3_1, Q4_0, Q4_1, Q5_0, Q5_1, Q6_0, Q6_1, Q8_0, Q8_1,
    BF16 = 12, F16 = 13, NONE = 14
};

bool is_lowbit(int f) { return f >= Q2_0 && f <= Q8_1; }
bool is_tail(int f) { return f == Q8_0 || f == BF16 || f == F16; }

int fmt_bits(int f) {
    static const int b[12] = {2, 2, 3, 3, 4, 4, 5, 5, 6, 6, 8, 8};
    if (is_lowbit(f)) return b[f];
    if (f == BF16 || f == F16) return 16;
    return 0;
}
bool fmt_asym(int f) { return is_lowbit(f) && (f % 2 == 1); }

// Bytes of one 32-value block. qX_0: fp16 scale + 32 X-bit codes = 2 + 4X;
// qX_1: fp16 scale + fp16 min + codes = 4 + 4X ([KVBENCH] table: q8_0 = 34/64 of
// bf16, q6_0 = 26/64, q5_1 = 24/64). bf16/f16: 32 x 2 bytes.
int block_bytes(int f) {
    if (is_lowbit(f)) return (fmt_asym(f) ? 4 : 2) + 4 * fmt_bits(f);
    if (f == BF16 || f == F16) return 64;
    return 0;
}

// Code planes, low bits first (READING: power-of-two planes so every element of a
// plane sits inside one byte). Returns the plane count; widths in w[0..1].
int planes(int bitsX, int w[2]) {
    switch (bitsX) {
        case 8: w[0] = 8; return 1;
        case 6: w[0] = 4; w[1] = 2; return 2;
        case 5: w[0] = 4; w[1] = 1; return 2;
        case 4: w[0] = 4; return 1;
        case 3: w[0] = 2; w[1] = 1; return 2;
        case 2: w[0] = 2; return 1;
    }
    return 0;
}

// ---------------------------------------------------------------------------
// IEEE-754 binary16 / bfloat16 conversion, written from the format definitions:
// round the exact value to the nearest representable number, ties to the one
// with an even last significand bit; overflow rounds to infinity.
// ---------------------------------------------------------------------------
uint32_t f32_bits(float x) { uint32_t u; std::memcpy(&u, &x, 4); return u; }
float bits_f32(uint32_t u) { float x; std::memcpy(&x, &u, 4); return x; }

// Generic: round |x| (finite, nonzero) to a format with `man_bits` stored
// mantissa bits, minimum normal exponent emin, and maximum biased exponent
// emax_field (all-ones is inf/nan). Returns the magnitude bits of the result.
uint32_t round_to_small_float(uint32_t mag_bits, int man_bits, int emin, int emax_field) {
    // exact value = M * 2^E with M a 24-bit (or smaller) integer
    int e32 = (int)(mag_bits >> 23);
    uint64_t M = mag_bits & 0x7fffff;
    int E;
    if (e32 == 0) { E = -149; } else { M |= 0x800000; E = e32 - 150; }
    int msb = 63 - __builtin_clzll(M);
    int p = msb + E;                       // value in [2^p, 2^(p+1))
    int Eq = std::max(p - man_bits, emin - man_bits);  // quantum exponent
    int shift = Eq - E;
    uint64_t r;
    if (shift <= 0) {
        r = M << (-shift);
    } else if (shift >= 64) {
        r = 0;                             // far below half a quantum
    } else {
        r = M >> shift;
        uint64_t rem = M & ((1ull << shift) - 1);
        uint64_t half = 1ull << (shift - 1);
        if (rem > half || (rem == half && (r & 1))) r += 1;
    }
    const uint64_t one = 1ull << man_bits;  // implicit bit position
    if (r == 2 * one) { r = one; Eq += 1; }
    if (r >= one) {
        int efield = Eq + man_bits - emin + 1;   // biased exponent
        if (efield >= emax_field) return (uint32_t)emax_field << man_bits;  // inf
        return ((uint32_t)efield << man_bits) | (uint32_t)(r - one);
    }
    return (uint32_t)r;                    // subnormal or zero
}

uint16_t f32_to_f16(float x) {
    uint32_t u = f32_bits(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000);
    uint32_t mag = u & 0x7fffffff;
    if (mag >= 0x7f800000) {               // inf or nan
        if (mag == 0x7f800000) return sign | 0x7c00;
        return sign | 0x7e00;
    }
    if (mag == 0) return sign;
    return sign | (uint16_t)round_to_small_float(mag, 10, -14, 31);
}

float f16_to_f32(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) v = std::ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = std::ldexp((double)(1024 + m), e - 25);
    return (float)(sign ? -v : v);
}

uint16_t f32_to_bf16(float x) {
    uint32_t u = f32_bits(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000);
    uint32_t mag = u & 0x7fffffff;
    if (mag >= 0x7f800000) {
        if (mag == 0x7f800000) return sign | 0x7f80;
        return sign | 0x7fc0;
    }
    if (mag == 0) return sign;
    return sign | (uint16_t)round_to_small_float(mag, 7, -126, 255);
}

float bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

// fp16 with saturation to +-65504 before rounding (READING: a block scale never
// becomes infinite).
uint16_t f32_to_f16_sat(float x) {
    if (x > 65504.0f) x = 65504.0f;
    if (x < -65504.0f) x = -65504.0f;
    return f32_to_f16(x);
}

// Round half away from zero, then clamp: the defined rounding of the cache codes.
float rhaz(float x) { return std::roundf(x); }

// ---------------------------------------------------------------------------
// Block quantization of k values (k = 32 in the cache; smaller k only in tests).
//
// qX_0 (symmetric, READING generalising the q8_0 "absmax/127" rule):
//   qmax = 2^(X-1) - 1, a = max|x|, d = fp16(a / qmax),
//   q_i = clamp(rhaz(x_i / d), -qmax, qmax), stored u_i = q_i + 2^(X-1);
//   d == 0 stores q_i = 0. Dequant: d * (u - 2^(X-1)).
// qX_1 (asymmetric, READING): lo = min x, hi = max x, d = fp16((hi - lo) / (2^X - 1)),
//   m = fp16(lo), u_i = clamp(rhaz((x_i - m) / d), 0, 2^X - 1); d == 0 stores u = 0.
//   Dequant: d * u + m.
// All arithmetic is float32 with IEEE round-to-nearest; division is a true division.
// ---------------------------------------------------------------------------
void quantize_codes(int f, const float* x, int k, uint8_t* u, uint16_t* d16, uint16_t* m16) {
    const int X = fmt_bits(f);
    if (!fmt_asym(f)) {
        const int qmax = (1 << (X - 1)) - 1;
        const int off = 1 << (X - 1);
        float a = 0.0f;
        for (int i = 0; i < k; ++i) a = std::max(a, std::fabs(x[i]));
        float d32 = a / (float)qmax;
        uint16_t dh = f32_to_f16_sat(d32);
        float d = f16_to_f32(dh);
        *d16 = dh;
        *m16 = 0;
        for (int i = 0; i < k; ++i) {
            int q = 0;
            if (d != 0.0f) {
                float r = rhaz(x[i] / d);
                if (r > (float)qmax) r = (float)qmax;
                if (r < (float)-qmax) r = (float)-qmax;
                q = (int)r;
            }
            u[i] = (uint8_t)(q + off);
        }
    } else {
        const int umax = (1 << X) - 1;
        float lo = x[0], hi = x[0];
        for (int i = 1; i < k; ++i) { lo = std::min(lo, x[i]); hi = std::max(hi, x[i]); }
        float d32 = (hi - lo) / (float)umax;
        uint16_t dh = f32_to_f16_sat(d32);
        uint16_t mh = f32_to_f16_sat(lo);
        float d = f16_to_f32(dh), m = f16_to_f32(mh);
        *d16 = dh;
        *m16 = mh;
        for (int i = 0; i < k; ++i) {
            int q = 0;
            if (d != 0.0f) {
                float r = rhaz((x[i] - m) / d);
                if (r > (float)umax) r = (float)umax;
                if (r < 0.0f) r = 0.0f;
                q = (int)r;
            }
            u[i] = (uint8_t)q;
        }
    }
}

float dequant_code(int f, uint16_t d16, uint16_t m16, int u) {
    const int X = fmt_bits(f);
    float d = f16_to_f32(d16);
    if (!fmt_asym(f)) return d * (float)(u - (1 << (X - 1)));   // exact product
    return d * (float)u + f16_to_f32(m16);                      // exact product, one rounded add
}

// Serialise 32 codes + scale (+ min): d | [m] | plane0 | [plane1], little endian.
void pack_block(int f, const uint8_t* u, uint16_t d16, uint16_t m16, uint8_t* out) {
    const int X = fmt_bits(f);
    int w[2] = {0, 0};
    int np = planes(X, w);
    out[0] = (uint8_t)(d16 & 0xff);
    out[1] = (uint8_t)(d16 >> 8);
    uint8_t* p = out + 2;
    if (fmt_asym(f)) { p[0] = (uint8_t)(m16 & 0xff); p[1] = (uint8_t)(m16 >> 8); p += 2; }
    int lowbit = 0;
    for (int pl = 0; pl < np; ++pl) {
        const int wb = w[pl];
        std::memset(p, 0, 4 * wb);
        for (int i = 0; i < 32; ++i) {
            int field = (u[i] >> lowbit) & ((1 << wb) - 1);
            int bit = wb * i;                      // bit offset in the plane's bitstream
            p[bit / 8] |= (uint8_t)(field << (bit % 8));
        }
        p += 4 * wb;
        lowbit += wb;
    }
}

void unpack_block(int f, const uint8_t* in, uint8_t* u, uint16_t* d16, uint16_t* m16) {
    const int X = fmt_bits(f);
    int w[2] = {0, 0};
    int np = planes(X, w);
    *d16 = (uint16_t)(in[0] | (in[1] << 8));
    const uint8_t* p = in + 2;
    *m16 = 0;
    if (fmt_asym(f)) { *m16 = (uint16_t)(p[0] | (p[1] << 8)); p += 2; }
    for (int i = 0; i < 32; ++i) u[i] = 0;
    int lowbit = 0;
    for (int pl = 0; pl < np; ++pl) {
        const int wb = w[pl];
        for (int i = 0; i < 32; ++i) {
            int bit = wb * i;
            int field = (p[bit / 8] >> (bit % 8)) & ((1 << wb) - 1);
            u[i] = (uint8_t)(u[i] | (field << lowbit));
        }
        p += 4 * wb;
        lowbit += wb;
    }
}

// One row of D values (D % 32 == 0) in format f -> D/32 canonical blocks.
void quantize_row(int f, const float* x, int D, uint8_t* out) {
    const int bb = block_bytes(f);
    for (int blk = 0; blk < D / 32; ++blk) {
        const float* xb = x + 32 * blk;
        uint8_t* ob = out + (size_t)bb * blk;
        if (f == BF16 || f == F16) {
            for (int i = 0; i < 32; ++i) {
                uint16_t h = (f == BF16) ? f32_to_bf16(xb[i]) : f32_to_f16(xb[i]);
                ob[2 * i] = (uint8_t)(h & 0xff);
                ob[2 * i + 1] = (uint8_t)(h >> 8);
            }
        } else {
            uint8_t u[32];
            uint16_t d16, m16;
            quantize_codes(f, xb, 32, u, &d16, &m16);
            pack_block(f, u, d16, m16, ob);
        }
    }
}

void dequant_row(int f, const uint8_t* in, int D, float* x) {
    const int bb = block_bytes(f);
    for (int blk = 0; blk < D / 32; ++blk) {
        const uint8_t* ib = in + (size_t)bb * blk;
        float* xb = x + 32 * blk;
        if (f == BF16 || f == F16) {
            for (int i = 0; i < 32; ++i) {
                uint16_t h = (uint16_t)(ib[2 * i] | (ib[2 * i + 1] << 8));
                xb[i] = (f == BF16) ? bf16_to_f32(h) : f16_to_f32(h);
            }
        } else {
            uint8_t u[32];
            uint16_t d16, m16;
            unpack_block(f, ib, u, &d16, &m16);
            for (int i = 0; i < 32; ++i) xb[i] = dequant_code(f, d16, m16, u[i]);
        }
    }
}

// ---------------------------------------------------------------------------
// The cache (READING of [HARDNUM] "KV cache low-bit storage" + "Reddit reactions"
// and [BEELLAMA] "KV cache precision tail"):
//  * a full-length low-bit main store per (layer, batch, kv head, K|V), one row per
//    position, plus a separate W-row ring in the tail format ([BEELLAMA] KV-MiB table:
//    the tail adds W rows of bf16 on top of the low-bit store);
//  * after any append the last min(n, W) positions live in ring slot pos mod W,
//    positions [0, n - W) in the main store;
//  * a position leaving the window is requantized from its ring entry
//    ("blocks must be requantized when the window boundary moves", [HARDNUM]
//    "Reddit reactions"): low = Q_low(deq_tail(ring entry)).
// KVarN ([BEELLAMA] names it; READING fixed by the workload definition):
//  s_c = fp32(sqrt(S/T + eps)), S = sum over the first T tokens of x^2 in fp64 with a
//  fixed pairwise tree; blocks quantize x / s_c; dequant multiplies by s_c.
// Per-channel K ([HARDNUM] "Reddit reactions": quantizing K along the token axis, as
// KIVI does, instead of 32 values per token; READING of its details):
//  * a K block is 32 consecutive positions of one channel: group g of channel c holds
//    the values of positions 32g .. 32g + 31, quantized with the same qX_0 / qX_1 rule;
//  * the value of a position entering the K store is the same as for per-token blocks
//    (deq_tail(Q_tail(x)) with a ring, x without one);
//  * a group is quantized when its last position enters the K store (leaves the window);
//    until then the positions that have entered are held exactly (fp32) in a 32-row
//    pending buffer, slot pos mod 32, and attention reads them from there;
//  * V keeps per-token blocks; per-channel K is not combined with KVarN.
// ---------------------------------------------------------------------------
struct Cache {
    int L, B, H, Hq, D;
    int64_t max_ctx;
    int kf, vf, tf, W;
    int kvarn, calib;
    int kivi;                                     // per-channel (token-axis) K blocks
    double eps;
    std::vector<int64_t> n;                       // per layer
    std::vector<std::vector<uint8_t>> main_;      // [L][B][H][2] rows of max_ctx
    std::vector<std::vector<uint8_t>> ring;       // [L][B][H][2] rows of W
    std::vector<float> s;                         // [L][B][H][2][D]
    std::vector<char> s_set;                      // [L]
    std::vector<std::vector<float>> pend;         // per-channel K: [L][B][H] 32 x D pending values

    size_t unit(int l, int b, int h, int kv) const { return (((size_t)l * B + b) * H + h) * 2 + kv; }
    size_t head(int l, int b, int h) const { return ((size_t)l * B + b) * H + h; }
    // per-channel K: block of channel c of group g, canonical bytes
    size_t group_block(int64_t g, int c) const { return ((size_t)g * D + c) * block_bytes(kf); }
    int low_fmt(int kv) const { return kv ? vf : kf; }
    size_t row_bytes(int f) const { return (size_t)block_bytes(f) * (D / 32); }
};

enum Status { OK = 0, ERR_INVALID_ARG = 1, ERR_UNSUPPORTED_FMT = 2, ERR_CAPACITY = 3,
              ERR_CALIBRATION = 4, ERR_EMPTY = 5 };

template <class F>
void parallel_for(int64_t count, int nthreads, F fn) {
    if (nthreads <= 1 || count <= 1) { for (int64_t i = 0; i < count; ++i) fn(i); return; }
    nthreads = (int)std::min<int64_t>(nthreads, count);
    std::vector<std::thread> th;
    for (int t = 0; t < nthreads; ++t)
        th.emplace_back([&, t] { for (int64_t i = t; i < count; i += nthreads) fn(i); });
    for (auto& x : th) x.join();
}

// Normalise (KVarN) a row before low-bit quantization: y = x / s (fp32 division).
void kvarn_divide(const float* x, const float* s, int D, float* y) {
    for (int c = 0; c < D; ++c) y[c] = x[c] / s[c];
}

// Per-channel K: position pos enters the K store with values x (one per channel): it is
// held in pending slot pos mod 32; the last position of a group completes it, and every
// channel's 32 values are quantized into that channel's block of the group.
void store_kivi(Cache& C, int l, int b, int h, int64_t pos, const float* x) {
    const int D = C.D;
    float* pend = C.pend[C.head(l, b, h)].data();
    std::memcpy(pend + (size_t)(pos % 32) * D, x, sizeof(float) * D);
    if (pos % 32 != 31) return;
    const int64_t g = pos / 32;
    float vals[32];
    uint8_t codes[32];
    for (int c = 0; c < D; ++c) {
        for (int t = 0; t < 32; ++t) vals[t] = pend[(size_t)t * D + c];
        uint16_t d16 = 0, m16 = 0;
        quantize_codes(C.kf, vals, 32, codes, &d16, &m16);
        pack_block(C.kf, codes, d16, m16, &C.main_[C.unit(l, b, h, 0)][C.group_block(g, c)]);
    }
}

// Quantize one raw row x into the low-bit main store slot `pos`, via the tail
// format when the cache has a ring (the row then passed through the ring).
void store_low(Cache& C, int l, int b, int h, int kv, int64_t pos, const float* x_raw) {
    const int D = C.D;
    if (kv == 0 && C.kivi) { store_kivi(C, l, b, h, pos, x_raw); return; }
    const int f = C.low_fmt(kv);
    std::vector<float> y(x_raw, x_raw + D);
    if (C.kvarn) kvarn_divide(x_raw, &C.s[C.unit(l, b, h, kv) * D], D, y.data());
    quantize_row(f, y.data(), D, &C.main_[C.unit(l, b, h, kv)][(size_t)pos * C.row_bytes(f)]);
}

// Append one token's raw row at position p (the per-token definition; a chunk is
// the same as its tokens appended one at a time).
void append_token(Cache& C, int l, int b, int h, int kv, int64_t p, const float* x) {
    const int D = C.D;
    if (C.W == 0) { store_low(C, l, b, h, kv, p, x); return; }
    const size_t rb = C.row_bytes(C.tf);
    auto& ring = C.ring[C.unit(l, b, h, kv)];
    const int64_t slot = p % C.W;
    if (p >= C.W) {
        // position p - W leaves the window: requantize its ring entry
        std::vector<float> xt(D);
        dequant_row(C.tf, &ring[(size_t)slot * rb], D, xt.data());
        store_low(C, l, b, h, kv, p - C.W, xt.data());
    }
    quantize_row(C.tf, x, D, &ring[(size_t)slot * rb]);
}

// KVarN statistics from the first T tokens of [B][n][H][D] input x.
void kvarn_calibrate(Cache& C, int l, int kv, const float* x, int n_new) {
    const int B = C.B, H = C.H, D = C.D, T = C.calib;
    std::vector<double> a(T);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < D; ++c) {
                for (int t = 0; t < T; ++t) {
                    double v = (double)x[(((size_t)b * n_new + t) * H + h) * D + c];
                    a[t] = v * v;
                }
                for (int stride = T / 2; stride >= 1; stride /= 2)
                    for (int t = 0; t < stride; ++t) a[t] += a[t + stride];
                double m = a[0] / (double)T + C.eps;
                C.s[C.unit(l, b, h, kv) * D + c] = (float)std::sqrt(m);
            }
}

// Dequantized row of position pos as attention sees it.
void position_row(const Cache& C, int l, int b, int h, int kv, int64_t pos, int64_t n, float* out) {
    const int D = C.D;
    const size_t u = C.unit(l, b, h, kv);
    if (C.W > 0 && pos >= n - C.W) {
        dequant_row(C.tf, &C.ring[u][(size_t)(pos % C.W) * C.row_bytes(C.tf)], D, out);
        return;
    }
    if (kv == 0 && C.kivi) {
        // positions below the window: in a completed group, or still pending
        const int64_t in_store = C.W > 0 ? std::max<int64_t>(0, n - C.W) : n;
        if (pos >= in_store / 32 * 32) {
            const float* pend = C.pend[C.head(l, b, h)].data();
            std::memcpy(out, pend + (size_t)(pos % 32) * D, sizeof(float) * D);
            return;
        }
        uint8_t codes[32];
        for (int c = 0; c < D; ++c) {
            uint16_t d16 = 0, m16 = 0;
            unpack_block(C.kf, &C.main_[u][C.group_block(pos / 32, c)], codes, &d16, &m16);
            out[c] = dequant_code(C.kf, d16, m16, codes[pos % 32]);
        }
        return;
    }
    const int f = C.low_fmt(kv);
    dequant_row(f, &C.main_[u][(size_t)pos * C.row_bytes(f)], D, out);
    if (C.kvarn) {
        const float* s = &C.s[u * D];
        for (int c = 0; c < D; ++c) out[c] = s[c] * out[c];
    }
}

// Exact softmax attention of one query row (all G heads of kv head h) over
// positions [0, t_end): s_t = scale * sum_c q_c K_tc in fp64, p = exp(s - max),
// o = sum_t p_t V_t / sum_t p_t, rounded to fp32.
void attend_rows(const Cache& C, int l, int b, int h, int64_t n, int64_t t_end,
                 const float* const* qs, int G, float scale, float* const* outs) {
    const int D = C.D;
    std::vector<double> sc((size_t)G * t_end);
    std::vector<float> row(D);
    for (int64_t t = 0; t < t_end; ++t) {
        position_row(C, l, b, h, 0, t, n, row.data());
        for (int g = 0; g < G; ++g) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c) acc += (double)qs[g][c] * (double)row[c];
            sc[(size_t)g * t_end + t] = (double)scale * acc;
        }
    }
    std::vector<double> mx(G, -INFINITY), den(G, 0.0), o((size_t)G * D, 0.0);
    for (int g = 0; g < G; ++g)
        for (int64_t t = 0; t < t_end; ++t) mx[g] = std::max(mx[g], sc[(size_t)g * t_end + t]);
    for (int64_t t = 0; t < t_end; ++t) {
        position_row(C, l, b, h, 1, t, n, row.data());
        for (int g = 0; g < G; ++g) {
            double p = std::exp(sc[(size_t)g * t_end + t] - mx[g]);
            den[g] += p;
            for (int c = 0; c < D; ++c) o[(size_t)g * D + c] += p * (double)row[c];
        }
    }
    for (int g = 0; g < G; ++g)
        for (int c = 0; c < D; ++c) outs[g][c] = (float)(o[(size_t)g * D + c] / den[g]);
}

// Softmax attention of one query row (all G heads of kv head h) over an explicit list of
// positions (the index-gather decode: [OFFLOAD], the paragraph on the QSA indexer choosing a
// budget of 2,048 positions per step). READING: entries outside [0, n) are skipped; the
// others enter in list order, a repeated position counting once per entry; with no valid
// entry the output is zero. Arithmetic as in attend_rows: fp64 scores, exp(s - max), fp64
// sums, rounded to fp32.
void attend_list(const Cache& C, int l, int b, int h, int64_t n, const int32_t* list, int k,
                 const float* const* qs, int G, float scale, float* const* outs) {
    const int D = C.D;
    std::vector<int64_t> pos;
    for (int j = 0; j < k; ++j)
        if (list[j] >= 0 && list[j] < n) pos.push_back(list[j]);
    const size_t m = pos.size();
    if (m == 0) {
        for (int g = 0; g < G; ++g)
            for (int c = 0; c < D; ++c) outs[g][c] = 0.0f;
        return;
    }
    std::vector<double> sc((size_t)G * m);
    std::vector<float> row(D);
    for (size_t j = 0; j < m; ++j) {
        position_row(C, l, b, h, 0, pos[j], n, row.data());
        for (int g = 0; g < G; ++g) {
            double acc = 0.0;
            for (int c = 0; c < D; ++c) acc += (double)qs[g][c] * (double)row[c];
            sc[(size_t)g * m + j] = (double)scale * acc;
        }
    }
    std::vector<double> mx(G, -INFINITY), den(G, 0.0), o((size_t)G * D, 0.0);
    for (int g = 0; g < G; ++g)
        for (size_t j = 0; j < m; ++j) mx[g] = std::max(mx[g], sc[(size_t)g * m + j]);
    for (size_t j = 0; j < m; ++j) {
        position_row(C, l, b, h, 1, pos[j], n, row.data());
        for (int g = 0; g < G; ++g) {
            double p = std::exp(sc[(size_t)g * m + j] - mx[g]);
            den[g] += p;
            for (int c = 0; c < D; ++c) o[(size_t)g * D + c] += p * (double)row[c];
        }
    }
    for (int g = 0; g < G; ++g)
        for (int c = 0; c < D; ++c) outs[g][c] = (float)(o[(size_t)g * D + c] / den[g]);
}

}  // namespace

// ===========================================================================
// C ABI of the oracle (ctypes)
// ===========================================================================
extern "C" {

int orc_fmt_bits(int f) { return fmt_bits(f); }
int orc_fmt_asym(int f) { return fmt_asym(f) ? 1 : 0; }
int orc_block_bytes(int f) { return block_bytes(f); }

// Element-wise conversions; threads only split the index range.
void orc_f32_to_f16_array(const float* x, uint16_t* y, int64_t n) {
    const int64_t parts = 16;
    parallel_for(parts, 8, [&](int64_t p) {
        for (int64_t i = n * p / parts; i < n * (p + 1) / parts; ++i) y[i] = f32_to_f16(x[i]);
    });
}
void orc_f32_to_bf16_array(const float* x, uint16_t* y, int64_t n) {
    const int64_t parts = 16;
    parallel_for(parts, 8, [&](int64_t p) {
        for (int64_t i = n * p / parts; i < n * (p + 1) / parts; ++i) y[i] = f32_to_bf16(x[i]);
    });
}
void orc_f16_to_f32_array(const uint16_t* x, float* y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = f16_to_f32(x[i]);
}

// Quantize k values (block length k; 32 in the cache). codes: k bytes.
int orc_quantize_codes(int f, const float* x, int k, uint8_t* codes, uint16_t* d16, uint16_t* m16) {
    if (!is_lowbit(f) || k < 1 || k > 32) return ERR_INVALID_ARG;
    quantize_codes(f, x, k, codes, d16, m16);
    return OK;
}
float orc_dequant_code(int f, uint16_t d16, uint16_t m16, int u) { return dequant_code(f, d16, m16, u); }

int orc_pack_block(int f, const uint8_t* codes, uint16_t d16, uint16_t m16, uint8_t* out) {
    if (!is_lowbit(f)) return ERR_INVALID_ARG;
    pack_block(f, codes, d16, m16, out);
    return OK;
}
int orc_unpack_block(int f, const uint8_t* in, uint8_t* codes, uint16_t* d16, uint16_t* m16) {
    if (!is_lowbit(f)) return ERR_INVALID_ARG;
    unpack_block(f, in, codes, d16, m16);
    return OK;
}
int orc_quantize_row(int f, const float* x, int D, uint8_t* out) {
    if (!(is_lowbit(f) || f == BF16 || f == F16) || D % 32) return ERR_INVALID_ARG;
    quantize_row(f, x, D, out);
    return OK;
}
int orc_dequant_row(int f, const uint8_t* in, int D, float* out) {
    if (!(is_lowbit(f) || f == BF16 || f == F16) || D % 32) return ERR_INVALID_ARG;
    dequant_row(f, in, D, out);
    return OK;
}

void* orc_cache_new(int L, int B, int H, int Hq, int D, int64_t max_ctx, int kf, int vf, int tf,
                    int W, int kvarn, int calib, double eps, int kivi) {
    if (L < 1 || B < 1 || H < 1 || Hq < H || Hq % H || D < 32 || D % 32 || max_ctx < 1) return nullptr;
    if (kivi && kvarn) return nullptr;
    if (!is_lowbit(kf) || !is_lowbit(vf)) return nullptr;
    if ((W == 0) != (tf == NONE)) return nullptr;
    if (W < 0 || (W > 0 && !is_tail(tf))) return nullptr;
    if (kvarn && (calib < 2 || (calib & (calib - 1)))) return nullptr;
    Cache* C = new Cache();
    C->L = L; C->B = B; C->H = H; C->Hq = Hq; C->D = D; C->max_ctx = max_ctx;
    C->kf = kf; C->vf = vf; C->tf = tf; C->W = W;
    C->kvarn = kvarn; C->calib = calib; C->eps = eps; C->kivi = kivi ? 1 : 0;
    C->n.assign(L, 0);
    const size_t units = (size_t)L * B * H * 2;
    C->main_.resize(units);
    C->ring.resize(units);
    for (int l = 0; l < L; ++l)
        for (int b = 0; b < B; ++b)
            for (int h = 0; h < H; ++h)
                for (int kv = 0; kv < 2; ++kv) {
                    size_t u = C->unit(l, b, h, kv);
                    C->main_[u].assign((size_t)max_ctx * C->row_bytes(C->low_fmt(kv)), 0);
                    if (kv == 0 && C->kivi)   // whole groups of 32 positions
                        C->main_[u].assign((size_t)((max_ctx + 31) / 32) * C->group_block(1, 0), 0);
                    if (W > 0) C->ring[u].assign((size_t)W * C->row_bytes(tf), 0);
                }
    C->s.assign(units * D, 1.0f);
    if (C->kivi) C->pend.assign(units / 2, std::vector<float>((size_t)32 * D, 0.0f));
    C->s_set.assign(L, 0);
    return C;
}

void orc_cache_free(void* c) { delete (Cache*)c; }

int64_t orc_length(void* c, int l) { return ((Cache*)c)->n[l]; }

int orc_set_channel_scales(void* c, int l, const float* sK, const float* sV) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L || !C.kvarn) return ERR_INVALID_ARG;
    for (int b = 0; b < C.B; ++b)
        for (int h = 0; h < C.H; ++h)
            for (int d = 0; d < C.D; ++d) {
                C.s[C.unit(l, b, h, 0) * C.D + d] = sK[((size_t)b * C.H + h) * C.D + d];
                C.s[C.unit(l, b, h, 1) * C.D + d] = sV[((size_t)b * C.H + h) * C.D + d];
            }
    C.s_set[l] = 1;
    return OK;
}

int orc_get_channel_scales(void* c, int l, float* sK, float* sV) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L) return ERR_INVALID_ARG;
    for (int b = 0; b < C.B; ++b)
        for (int h = 0; h < C.H; ++h)
            for (int d = 0; d < C.D; ++d) {
                sK[((size_t)b * C.H + h) * C.D + d] = C.s[C.unit(l, b, h, 0) * C.D + d];
                sV[((size_t)b * C.H + h) * C.D + d] = C.s[C.unit(l, b, h, 1) * C.D + d];
            }
    return OK;
}

// k, v: fp32 [B][n_new][H][D].
int orc_append(void* c, int l, const float* k, const float* v, int n_new, int nthreads) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L || n_new < 0) return ERR_INVALID_ARG;
    if (C.n[l] + n_new > C.max_ctx) return ERR_CAPACITY;
    if (n_new == 0) return OK;
    if (C.kvarn && !C.s_set[l]) {
        if (C.n[l] != 0 || n_new < C.calib) return ERR_CALIBRATION;
        kvarn_calibrate(C, l, 0, k, n_new);
        kvarn_calibrate(C, l, 1, v, n_new);
        C.s_set[l] = 1;
    }
    const int64_t n0 = C.n[l];
    // (batch, kv head, K|V) units are independent; tokens go in order within a unit.
    parallel_for((int64_t)C.B * C.H * 2, nthreads, [&](int64_t u) {
        int kv = (int)(u % 2), h = (int)((u / 2) % C.H), b = (int)(u / (2 * C.H));
        const float* x = kv ? v : k;
        for (int t = 0; t < n_new; ++t)
            append_token(C, l, b, h, kv, n0 + t, x + (((size_t)b * n_new + t) * C.H + h) * C.D);
    });
    C.n[l] = n0 + n_new;
    return OK;
}

// Canonical bytes of rows [pos0, pos0 + count) of one (layer, b, h, K|V):
// region 0 = main-store positions, region 1 = ring slots.
int orc_export(void* c, int l, int b, int h, int kv, int region, int64_t pos0, int64_t count, uint8_t* dst) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L || b < 0 || b >= C.B || h < 0 || h >= C.H || kv < 0 || kv > 1) return ERR_INVALID_ARG;
    const size_t u = C.unit(l, b, h, kv);
    if (region == 0 && kv == 0 && C.kivi) {
        // per-channel K: groups pos0 .. pos0 + count - 1, each its D channel blocks in order
        if (pos0 < 0 || count < 0 || pos0 + count > (C.max_ctx + 31) / 32) return ERR_INVALID_ARG;
        std::memcpy(dst, &C.main_[u][C.group_block(pos0, 0)], (size_t)count * C.group_block(1, 0));
        return OK;
    }
    if (region == 2) {
        // per-channel K pending slots pos0 .. pos0 + count - 1 as fp32 rows of D values
        if (!C.kivi || kv != 0 || pos0 < 0 || count < 0 || pos0 + count > 32) return ERR_INVALID_ARG;
        std::memcpy(dst, &C.pend[C.head(l, b, h)][(size_t)pos0 * C.D], (size_t)count * C.D * sizeof(float));
        return OK;
    }
    if (region == 0) {
        if (pos0 < 0 || count < 0 || pos0 + count > C.max_ctx) return ERR_INVALID_ARG;
        size_t rb = C.row_bytes(C.low_fmt(kv));
        std::memcpy(dst, &C.main_[u][(size_t)pos0 * rb], (size_t)count * rb);
        return OK;
    }
    if (region == 1) {
        if (C.W == 0 || pos0 < 0 || count < 0 || pos0 + count > C.W) return ERR_INVALID_ARG;
        size_t rb = C.row_bytes(C.tf);
        std::memcpy(dst, &C.ring[u][(size_t)pos0 * rb], (size_t)count * rb);
        return OK;
    }
    return ERR_INVALID_ARG;
}

// Dequantized row at a position, as attention reads it (out: D floats).
int orc_position_row(void* c, int l, int b, int h, int kv, int64_t pos, float* out) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L || pos < 0 || pos >= C.n[l]) return ERR_INVALID_ARG;
    position_row(C, l, b, h, kv, pos, C.n[l], out);
    return OK;
}

// Decode attention over all n cached positions. q, out: fp32 [B][Hq][D].
// Query head hq reads kv head hq / G (READING: contiguous grouping).
int orc_decode(void* c, int l, const float* q, float scale, float* out, int nthreads) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L) return ERR_INVALID_ARG;
    const int64_t n = C.n[l];
    if (n == 0) return ERR_EMPTY;
    const int G = C.Hq / C.H;
    parallel_for((int64_t)C.B * C.H, nthreads, [&](int64_t u) {
        int b = (int)(u / C.H), h = (int)(u % C.H);
        std::vector<const float*> qs(G);
        std::vector<float*> os(G);
        for (int g = 0; g < G; ++g) {
            size_t off = ((size_t)b * C.Hq + h * G + g) * C.D;
            qs[g] = q + off;
            os[g] = out + off;
        }
        attend_rows(C, l, b, h, n, n, qs.data(), G, scale, os.data());
    });
    return OK;
}

// Index-gather decode: like orc_decode, but each (batch, kv head) attends only to the k
// positions listed in idx[b][h][0..k) (see attend_list for the reading of the list).
// q, out: fp32 [B][Hq][D]; idx: int32 [B][H][k].
int orc_decode_indexed(void* c, int l, const float* q, float scale, const int32_t* idx, int k, float* out,
                       int nthreads) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L || k < 1) return ERR_INVALID_ARG;
    const int64_t n = C.n[l];
    if (n == 0) return ERR_EMPTY;
    const int G = C.Hq / C.H;
    parallel_for((int64_t)C.B * C.H, nthreads, [&](int64_t u) {
        int b = (int)(u / C.H), h = (int)(u % C.H);
        std::vector<const float*> qs(G);
        std::vector<float*> os(G);
        for (int g = 0; g < G; ++g) {
            size_t off = ((size_t)b * C.Hq + h * G + g) * C.D;
            qs[g] = q + off;
            os[g] = out + off;
        }
        attend_list(C, l, b, h, n, idx + (size_t)u * k, k, qs.data(), G, scale, os.data());
    });
    return OK;
}

// Causal prefill attention of the last n_chunk appended rows over the post-append
// cache: chunk row i sits at position n - n_chunk + i and attends to t <= that.
// q, out: fp32 [B][n_chunk][Hq][D]. rows (optional, n_rows entries) restricts the
// computed chunk rows; other rows of out are left untouched.
int orc_prefill(void* c, int l, const float* q, int n_chunk, float scale, float* out,
                const int32_t* rows, int n_rows, int nthreads) {
    Cache& C = *(Cache*)c;
    if (l < 0 || l >= C.L) return ERR_INVALID_ARG;
    const int64_t n = C.n[l];
    if (n_chunk < 1 || n_chunk > n) return n == 0 ? ERR_EMPTY : ERR_INVALID_ARG;
    const int G = C.Hq / C.H;
    const int R = rows ? n_rows : n_chunk;
    if (rows)
        for (int r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= n_chunk) return ERR_INVALID_ARG;
    parallel_for((int64_t)C.B * C.H * R, nthreads, [&](int64_t u) {
        int r = (int)(u % R);
        int h = (int)((u / R) % C.H);
        int b = (int)(u / ((int64_t)R * C.H));
        int i = rows ? rows[r] : r;
        int64_t pos = n - n_chunk + i;
        std::vector<const float*> qs(G);
        std::vector<float*> os(G);
        for (int g = 0; g < G; ++g) {
            size_t off = (((size_t)b * n_chunk + i) * C.Hq + h * G + g) * C.D;
            qs[g] = q + off;
            os[g] = out + off;
        }
        attend_rows(C, l, b, h, n, pos + 1, qs.data(), G, scale, os.data());
    });
    return OK;
}

}  // extern "C"
