// kvq_append.cu -- quantize-on-append, tail-ring eviction with requantization, and the
// KVarN channel-statistics pass.
//
// One warp owns one (position, batch, kv head, K|V) row of D = 32*CPL channels; lane l
// holds channels [l*CPL, (l+1)*CPL), so a 32-value block spans 32/CPL lanes and its
// max / min reduce with xor shuffles inside that lane group. Inputs are read with
// 16-byte loads, codes are packed in registers and written as whole words per lane.
//
// Block rules ([HARDNUM] "Reddit reactions": 32 values per token block; byte counts
// from the [KVBENCH] cache-size table):
//   qX_0: d = fp16(absmax / (2^(X-1)-1)) (saturating), q = clamp(rhaz(x / d)), u = q + 2^(X-1)
//   qX_1: d = fp16((max - min) / (2^X - 1)), m = fp16(min), u = clamp(rhaz((x - m) / d))
// with the IEEE float32 quotient (computed without a division where that is provably
// identical, see div_range and round_codes) and round-half-away-from-zero (roundf).
//
// Ring ([HARDNUM] "KV cache low-bit storage": the last 2,048 positions in an 8-bit ring;
// [BEELLAMA] precision tail): after an append of C rows to a cache of n, positions
// [n+C-W, n+C) sit in ring slot pos mod W. A new position that ends inside the window
// takes its slot: the warp first requantizes the slot's old occupant (the unique
// position q in [n-W, n) with q = pos mod W) into the low-bit store, then writes the new
// row. Every evicted position's slot receives exactly one such new row, and slots are
// distinct across warps, so no two warps touch one slot. Positions that enter and leave
// within the append go to the low-bit store directly, through the tail rounding.
#include "kvq_rowio.cuh"

#include <algorithm>
#include <type_traits>

namespace kvq {
namespace {

constexpr int WARPS_PER_CTA = 8;

template <int CPL>
struct Lanes {
    static constexpr int LPB = 32 / CPL;   // lanes per 32-value block
};

// fl(1 / (2^k - 1)), k = 0..8 (entry 0 unused)
__constant__ float c_rcp_range[9] = {0.f, 0x1p+0f, 0x1.555556p-2f, 0x1.24924ap-3f, 0x1.111112p-4f,
                                     0x1.08421p-5f, 0x1.041042p-6f, 0x1.020408p-7f, 0x1.010102p-8f};

// fl(a / (2^k - 1)) for a >= 0, k = 1..8, without a division: q = fl(a * y) with
// y = fl(1 / b) is refined once with the exact residual a - q * b (Markstein's division by
// a constant). Checked exhaustively against IEEE division for every non-negative fp32 a and
// every b = 2^k - 1 the formats use. An infinite a gives NaN, which the saturating clamp
// that follows maps to the same value as the quotient inf.
__device__ __forceinline__ float div_range(float a, int k) {
    const float b = (float)((1 << k) - 1);
    const float y = c_rcp_range[k];
    const float q = __fmul_rn(a, y);
    const float r = __fmaf_rn(-q, b, a);
    return __fmaf_rn(r, y, q);
}

// hardware reciprocal (at most 1 ulp from 1/d)
__device__ __forceinline__ float rcp_approx(float d) {
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

constexpr float MAGIC = 12582912.0f;          // 1.5 * 2^23: adding it rounds |r| < 2^22 to an integer
constexpr int MAGIC_BITS = 0x4B400000;         // bit pattern of MAGIC

// Codes rhaz(fl((x_j - m) / d)) clamped to [lo, hi], for d > 0 (all zero when d == 0), returned as
// t_j = MAGIC + code (so code = bits(t_j) - MAGIC_BITS and the code as a float is t_j - MAGIC).
// r = (x - m) * rd with rd within 1 ulp of 1/d is within 2 * 2^-23 * |r| of fl((x - m) / d).
// Clamping to integer bounds commutes with rounding, and after it |r| <= lim = max(|lo|, |hi|),
// so unless r lies within 4e-7 * lim of a half-integer both have the same nearest integer
// (which is then not a tie) and the rounding add gives it. A lane with such a near-tie redoes its values from the correctly
// rounded IEEE quotient, once for all CPL values.
template <int CPL, bool ASYM>
__device__ __forceinline__ void round_codes(const float (&x)[CPL], float d, float m, float lo, float hi,
                                            float (&t)[CPL]) {
    const float rd = d != 0.f ? rcp_approx(d) : 0.f;
    const float tol = 4e-7f * fmaxf(-lo, hi);
    bool near = false;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const float v = ASYM ? __fsub_rn(x[j], m) : x[j];
        const float r = fminf(fmaxf(__fmul_rn(v, rd), lo), hi);
        t[j] = __fadd_rn(r, MAGIC);
        const float e = __fsub_rn(r, __fsub_rn(t[j], MAGIC));     // exact, |e| <= 1/2
        near |= fabsf(__fsub_rn(fabsf(e), 0.5f)) <= tol;
    }
    if (near) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const float v = ASYM ? __fsub_rn(x[j], m) : x[j];
            t[j] = __fadd_rn(fminf(fmaxf(roundf(__fdiv_rn(v, d)), lo), hi), MAGIC);
        }
    }
}

// pack CPL codes (bits below W0 into plane 0, the next W1 bits into plane 1) and store
template <int CPL, int W0, int W1>
__device__ __forceinline__ void pack_store(uint8_t* p0, uint8_t* p1, int lane, const uint32_t (&u)[CPL]) {
    // 32-bit accumulators unless a lane's plane bits need 64
    using A0 = typename std::conditional<(CPL * W0 > 32), uint64_t, uint32_t>::type;
    using A1 = typename std::conditional<(CPL * W1 > 32), uint64_t, uint32_t>::type;
    A0 v0 = 0;
    A1 v1 = 0;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        v0 |= (A0)(u[j] & ((1u << W0) - 1)) << (j * W0);
        if constexpr (W1 > 0) v1 |= (A1)(u[j] >> W0) << (j * W1);
    }
    // a row of D = 32 * CPL channels has CPL blocks
    store_plane_bits<CPL>(p0, CPL, lane, W0, v0);
    if constexpr (W1 > 0) store_plane_bits<CPL>(p1, CPL, lane, W1, v1);
}

// Quantize this lane's CPL values into row `row` of format f (all lanes participate).
// Returns an upper bound of |stored value| over this lane's values (the block bound d*qmax,
// or |m| + d*umax, for block formats; the 16-bit rounding of |x| for bf16 / f16 rows).
template <int CPL>
__device__ __forceinline__ float store_row(uint8_t* __restrict__ row, const RowFmt& f, int lane,
                                           const float (&x)[CPL]) {
    constexpr int LPB = Lanes<CPL>::LPB;
    if (f.kind != 0) {
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) a = fmaxf(a, fabsf(x[j]));
        uint16_t h[CPL];
#pragma unroll
        for (int j = 0; j < CPL; ++j)
            h[j] = (f.kind == 1) ? __bfloat16_as_ushort(__float2bfloat16_rn(x[j]))
                                 : __half_as_ushort(__float2half_rn(x[j]));
        uint16_t* dst = reinterpret_cast<uint16_t*>(row) + lane * CPL;
        if constexpr (CPL == 8) {
            uint4 w;
            w.x = h[0] | ((uint32_t)h[1] << 16); w.y = h[2] | ((uint32_t)h[3] << 16);
            w.z = h[4] | ((uint32_t)h[5] << 16); w.w = h[6] | ((uint32_t)h[7] << 16);
            *reinterpret_cast<uint4*>(dst) = w;
        } else {
#pragma unroll
            for (int j = 0; j < CPL; ++j) dst[j] = h[j];
        }
        return a * 1.0078125f;          // a 16-bit rounding grows |x| by at most 2^-8
    }
    const int blk = (lane * CPL) >> 5;
    uint32_t u[CPL];
    uint16_t dh, mh = 0;
    float bound;
    if (!f.asym) {
        const int qmax = (1 << (f.bits - 1)) - 1;
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) a = fmaxf(a, fabsf(x[j]));
        a = group_max<LPB>(a);
        const float d32 = div_range(a, f.bits - 1);      // a / qmax
        dh = __half_as_ushort(__float2half_rn(fminf(d32, 65504.f)));
        const float d = __half2float(__ushort_as_half(dh));
        bound = d * (float)qmax;
        float t[CPL];
        round_codes<CPL, false>(x, d, 0.f, (float)-qmax, (float)qmax, t);
#pragma unroll
        for (int j = 0; j < CPL; ++j) u[j] = (uint32_t)(__float_as_int(t[j]) - (MAGIC_BITS - qmax - 1));
    } else {
        const int umax = (1 << f.bits) - 1;
        float lo = x[0], hi = x[0];
#pragma unroll
        for (int j = 1; j < CPL; ++j) { lo = fminf(lo, x[j]); hi = fmaxf(hi, x[j]); }
        lo = group_min<LPB>(lo);
        hi = group_max<LPB>(hi);
        const float d32 = div_range(__fsub_rn(hi, lo), f.bits);   // (hi - lo) / umax
        dh = __half_as_ushort(__float2half_rn(fminf(d32, 65504.f)));
        mh = __half_as_ushort(__float2half_rn(fminf(fmaxf(lo, -65504.f), 65504.f)));
        const float d = __half2float(__ushort_as_half(dh));
        const float m = __half2float(__ushort_as_half(mh));
        bound = fabsf(m) + d * (float)umax;
        float t[CPL];
        round_codes<CPL, true>(x, d, m, 0.f, (float)umax, t);
#pragma unroll
        for (int j = 0; j < CPL; ++j) u[j] = (uint32_t)(__float_as_int(t[j]) - MAGIC_BITS);
    }
    uint8_t* p0 = row + f.off_p0;
    uint8_t* p1 = row + f.off_p1;
    switch (f.bits) {
        case 8: pack_store<CPL, 8, 0>(p0, p1, lane, u); break;
        case 6: pack_store<CPL, 4, 2>(p0, p1, lane, u); break;
        case 5: pack_store<CPL, 4, 1>(p0, p1, lane, u); break;
        case 4: pack_store<CPL, 4, 0>(p0, p1, lane, u); break;
        case 3: pack_store<CPL, 2, 1>(p0, p1, lane, u); break;
        default: pack_store<CPL, 2, 0>(p0, p1, lane, u); break;
    }
    if ((lane % LPB) == 0) {
        reinterpret_cast<uint16_t*>(row)[blk] = dh;
        if (f.asym) reinterpret_cast<uint16_t*>(row + f.off_m)[blk] = mh;
    }
    return bound;
}

// Value bounds of the rows a warp stores: stored domain (block values) and dequantized
// domain (after the KVarN channel scale).
struct Bounds {
    float stored = 0.f, deq = 0.f;
    __device__ void add(float s, float d) { stored = fmaxf(stored, s); deq = fmaxf(deq, d); }
};

// Low-bit store of a raw row (KVarN: divide by the channel scales first).
template <int CPL>
__device__ __forceinline__ void store_low(uint8_t* row, const RowFmt& f, const float* __restrict__ s, int lane,
                                          float (&x)[CPL], Bounds& bd) {
    float smax = 1.f;
    if (s) {
        smax = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const float sc = s[lane * CPL + j];
            smax = fmaxf(smax, sc);
            x[j] = __fdiv_rn(x[j], sc);
        }
    }
    const float b = store_row<CPL>(row, f, lane, x);
    bd.add(b, b * smax);
}

// Raise the cache's per-head bounds to the maxima of the values a CTA of the append kernel
// stored (its warps share one (b, h, K|V)). Float bits of non-negative values order as
// unsigned integers (a NaN bound, which only a NaN input makes, orders above every finite
// one); the warps' maxima meet in shared memory and one thread raises the bounds with
// non-returning atomics, so no warp waits on a read of the bounds.
__device__ __forceinline__ void publish_bounds_cta(uint32_t* st, Bounds bd, uint32_t (*sb)[2]) {
    const uint32_t s_max = __reduce_max_sync(0xffffffffu, __float_as_uint(bd.stored));
    const uint32_t d_max = __reduce_max_sync(0xffffffffu, __float_as_uint(bd.deq));
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) { sb[warp][0] = s_max; sb[warp][1] = d_max; }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t a = 0, c = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) { a = max(a, sb[w][0]); c = max(c, sb[w][1]); }
        // margin for the fp32 rounding of dequantized values
        const uint32_t u0 = __float_as_uint(__uint_as_float(a) * 1.0009765625f);
        const uint32_t u1 = __float_as_uint(__uint_as_float(c) * 1.0009765625f);
        if (u0) atomicMax(st, u0);
        if (u1) atomicMax(st + 1, u1);
    }
}

// The values a ring round trip gives this lane's CPL values (the tail format's rounding,
// computed in registers; all lanes of the warp participate).
template <int CPL>
__device__ __forceinline__ void tail_round(const RowFmt& tail, const float (&x)[CPL], float (&t)[CPL]) {
    if (tail.kind == 1) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) t[j] = __bfloat162float(__float2bfloat16_rn(x[j]));
    } else if (tail.kind == 2) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) t[j] = __half2float(__float2half_rn(x[j]));
    } else {
        // q8_0 tail: symmetric 8-bit block quantization then exact dequantization
        constexpr int LPB = Lanes<CPL>::LPB;
        float a = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) a = fmaxf(a, fabsf(x[j]));
        a = group_max<LPB>(a);
        const float d32 = div_range(a, 7);               // a / 127
        const float d = __half2float(__float2half_rn(fminf(d32, 65504.f)));
        float c[CPL];
        round_codes<CPL, false>(x, d, 0.f, -127.f, 127.f, c);
#pragma unroll
        for (int j = 0; j < CPL; ++j) t[j] = __fmul_rn(d, __fsub_rn(c[j], MAGIC));
    }
}

// Per-channel K: a position whose group is not complete after this append enters the
// pending buffer (this lane's CPL values of its float32 row, slot pos mod 32); positions of
// groups completed by this append were quantized by kivi_group_kernel before this kernel.
template <int CPL>
__device__ __forceinline__ void kivi_enter(const LayerView& lv, uint32_t unit, long long pos, uint32_t done, int lane,
                                           const float (&x)[CPL]) {
    if (pos < (long long)done) return;
    float* dst = lv.pend + ((long long)unit * 32 + pos % 32) * lv.D + lane * CPL;
    if constexpr (CPL % 4 == 0) {
#pragma unroll
        for (int j = 0; j < CPL; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < CPL; ++j) dst[j] = x[j];
    }
}

// Ring slot arithmetic without a division: q = floor(x / W) = (x * m) >> 32 + s for x < 2^31,
// with s = ceil(log2 W) and m = ceil(2^(32 + s) / W) (Granlund and Montgomery's division by an
// invariant integer; the error term stays below 1 / W for 31-bit x), and n mod W from the host.
struct RingDiv {
    unsigned long long m;
    uint32_t s;
    uint32_t n_mod_w;
};

// One row of an append (warp-wide): quantize-on-append, ring eviction, requantization.
// Returns this lane's bounds of the values it stored (zero for per-channel K rows that only
// enter the pending buffer).
template <int CPL>
__device__ __forceinline__ Bounds append_row(const LayerView& lv, const float* __restrict__ k,
                                             const float* __restrict__ v, uint32_t n, uint32_t C,
                                             uint32_t kivi_done, const RingDiv& rd, uint32_t i, uint32_t kv,
                                             uint32_t h, uint32_t b, int lane) {
    const uint32_t row = b * C + i;
    const int D = lv.D;
    const float* src = (kv ? v : k) + ((long long)row * lv.H + h) * D;
    const RowFmt fl = kv ? lv.fmt[1] : lv.fmt[0];   // by value: no pointer into the parameters
    uint8_t* main = lv.main[kv] + (long long)(b * lv.H + h) * lv.main_region[kv];
    const float* s = lv.kvarn ? lv.scales + ((long long)(b * lv.H + h) * 2 + kv) * D : nullptr;
    const uint32_t p = n + i;
    const bool kivi = lv.kivi && kv == 0;            // per-channel K
    const uint32_t unit = b * lv.H + h;
    Bounds bd;
    float x[CPL];
    load_row_f32<CPL>(src, lane, x);

    if (lv.W == 0) {
        if (kivi) { kivi_enter<CPL>(lv, unit, p, kivi_done, lane, x); return bd; }
        store_low<CPL>(main + (long long)p * fl.stride, fl, s, lane, x, bd);
        return bd;
    }
    const uint32_t W = (uint32_t)lv.W;
    if (i + W < C) {
        // enters and leaves the window inside this append: tail rounding, then low-bit
        float t[CPL];
        tail_round<CPL>(lv.tail, x, t);
        if (kivi) { kivi_enter<CPL>(lv, unit, p, kivi_done, lane, t); return bd; }
        store_low<CPL>(main + (long long)p * fl.stride, fl, s, lane, t, bd);
        return bd;
    }
    // ends inside the window: evict the slot's old occupant, then take the slot
    uint8_t* ring = lv.ring[kv] + (long long)(b * lv.H + h) * lv.ring_region;
    const uint32_t im = i - W * (uint32_t)(((unsigned long long)i * rd.m) >> (32 + rd.s));   // i mod W
    uint32_t slot = rd.n_mod_w + im;                                                       // (n + i) mod W
    if (slot >= W) slot -= W;
    uint8_t* srow = ring + (long long)slot * lv.tail.stride;
    // old occupant: the position in [n - W, n) congruent to p = n + i modulo W
    const long long q = (long long)n - W + im;
    if (q >= 0) {
        float y[CPL];
        load_row_values<CPL>(srow, lv.tail, lane, y);
        __syncwarp();
        if (kivi) kivi_enter<CPL>(lv, unit, q, kivi_done, lane, y);
        else store_low<CPL>(main + (long long)q * fl.stride, fl, s, lane, y, bd);
    }
    __syncwarp();
    const float rb = store_row<CPL>(srow, lv.tail, lane, x);   // ring rows hold raw values
    bd.add(rb, rb);
    return bd;
}

// 6 CTAs (48 warps) per SM: the kernel is issue-bound, and the extra warps hide more latency
// than the few registers they cost (a handful of spills at 40 registers) take back
template <int CPL>
__global__ void __launch_bounds__(32 * WARPS_PER_CTA, 6)
append_kernel(LayerView lv, const float* __restrict__ k, const float* __restrict__ v, uint32_t n, uint32_t C,
              uint32_t kivi_done, RingDiv rd) {
    const int lane = threadIdx.x & 31;
    // warp = one row: position i of the append (consecutive warps, consecutive positions of the
    // same (b, h, K|V) region), blockIdx.y = 2 h + kv, blockIdx.z = b; the host keeps
    // positions below 2^31
    const uint32_t i = blockIdx.x * WARPS_PER_CTA + (threadIdx.x >> 5);
    const uint32_t kv = blockIdx.y & 1u;
    const uint32_t h = blockIdx.y >> 1;
    const uint32_t b = blockIdx.z;
    uint32_t* st = lv.stats + ((long long)(b * lv.H + h) * 2 + kv) * 2;
    __shared__ uint32_t sb[WARPS_PER_CTA][2];
    Bounds bd;
    if (i < C) bd = append_row<CPL>(lv, k, v, n, C, kivi_done, rd, i, kv, h, b, lane);
    publish_bounds_cta(st, bd, sb);   // every thread of the CTA takes part
}

// Per-channel K, groups completed by an append of C positions to a cache of n0: one CTA per
// (batch, kv head, group). Its 8 warps gather the group's 32 rows as they enter the K store
// (pending rows for positions that entered earlier, ring rows for positions leaving the
// window now, tail-rounded input rows for positions that enter and leave in this append,
// raw input rows without a ring) into shared memory; then thread c quantizes channel c's
// 32 values into its canonical block (same rules as a per-token block: absmax or min/max,
// division-free exact scale, rhaz codes) and writes it. Runs before append_kernel, which
// overwrites the ring slots and the pending rows.
template <int CPL>
__global__ void __launch_bounds__(256)
kivi_group_kernel(LayerView lv, const float* __restrict__ k, uint32_t n0, uint32_t C, uint32_t g0, uint32_t ngroups) {
    extern __shared__ float sg[];                        // [32][D]
    const int D = lv.D;
    const uint32_t unit = blockIdx.x / ngroups;          // b * H + h
    const uint32_t g = g0 + blockIdx.x % ngroups;
    const uint32_t b = unit / lv.H, h = unit % lv.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long W = lv.W;
    const long long entered_old = W ? max(0LL, (long long)n0 - W) : (long long)n0;
    for (int r = warp; r < 32; r += 8) {
        const long long p = 32LL * g + r;
        float x[CPL];
        if (p < entered_old) {
            const float* src = lv.pend + ((long long)unit * 32 + p % 32) * D + lane * CPL;
#pragma unroll
            for (int j = 0; j < CPL; ++j) x[j] = src[j];
        } else if (p < (long long)n0) {                  // leaves the ring now
            const uint8_t* srow = lv.ring[0] + (long long)unit * lv.ring_region + (p % W) * lv.tail.stride;
            load_row_values<CPL>(srow, lv.tail, lane, x);
        } else {
            const long long i = p - n0;
            float y[CPL];
            load_row_f32<CPL>(k + (((long long)b * C + i) * lv.H + h) * D, lane, y);
            if (W) tail_round<CPL>(lv.tail, y, x);
            else {
#pragma unroll
                for (int j = 0; j < CPL; ++j) x[j] = y[j];
            }
        }
#pragma unroll
        for (int j = 0; j < CPL; ++j) sg[r * D + lane * CPL + j] = x[j];
    }
    __syncthreads();
    const RowFmt f = lv.fmt[0];
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        float v[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = sg[t * D + c];
        uint32_t u[32];
        uint16_t dh, mh = 0;
        if (!f.asym) {
            const int qmax = (1 << (f.bits - 1)) - 1;
            float a = 0.f;
#pragma unroll
            for (int t = 0; t < 32; ++t) a = fmaxf(a, fabsf(v[t]));
            const float d32 = div_range(a, f.bits - 1);
            dh = __half_as_ushort(__float2half_rn(fminf(d32, 65504.f)));
            const float d = __half2float(__ushort_as_half(dh));
            float t[32];
            round_codes<32, false>(v, d, 0.f, (float)-qmax, (float)qmax, t);
#pragma unroll
            for (int j = 0; j < 32; ++j) u[j] = (uint32_t)(__float_as_int(t[j]) - (MAGIC_BITS - qmax - 1));
        } else {
            const int umax = (1 << f.bits) - 1;
            float lo = v[0], hi = v[0];
#pragma unroll
            for (int t = 1; t < 32; ++t) { lo = fminf(lo, v[t]); hi = fmaxf(hi, v[t]); }
            const float d32 = div_range(__fsub_rn(hi, lo), f.bits);
            dh = __half_as_ushort(__float2half_rn(fminf(d32, 65504.f)));
            mh = __half_as_ushort(__float2half_rn(fminf(fmaxf(lo, -65504.f), 65504.f)));
            const float d = __half2float(__ushort_as_half(dh));
            const float m = __half2float(__ushort_as_half(mh));
            float t[32];
            round_codes<32, true>(v, d, m, 0.f, (float)umax, t);
#pragma unroll
            for (int j = 0; j < 32; ++j) u[j] = (uint32_t)(__float_as_int(t[j]) - MAGIC_BITS);
        }
        // canonical block: d | [m] | plane0 (32 codes x w0 bits) | plane1 (32 codes x w1 bits)
        uint16_t* blk = reinterpret_cast<uint16_t*>(lv.main[0] + (long long)unit * lv.main_region[0] +
                                                    ((long long)g * D + c) * lv.kbb);
        int o = 0;
        blk[o++] = dh;
        if (f.asym) blk[o++] = mh;
        const int ws[2] = {f.w0, f.w1};
        for (int pl = 0; pl < 2; ++pl) {
            const int w = ws[pl];
            if (w == 0) break;
            const uint32_t mask = (1u << w) - 1;
            const int shift = pl ? f.w0 : 0;
            // 32 codes x w bits = 2w 16-bit words
            for (int q = 0; q < 2 * w; ++q) {
                uint32_t word = 0;
                const int per = 16 / w;                  // codes per 16-bit word
                for (int e = 0; e < per; ++e) word |= ((u[q * per + e] >> shift) & mask) << (e * w);
                blk[o++] = (uint16_t)word;
            }
        }
    }
}

// KVarN statistics: one CTA of T/2 threads per (b, h, K|V, channel group of 8);
// S_c = fixed pairwise tree over a[t] = x_t^2 (a[t] += a[t + stride], stride = T/2 .. 1)
// in float64; s_c = float(sqrt(S_c / T + eps)).
__global__ void calibrate_kernel(LayerView lv, const float* __restrict__ k, const float* __restrict__ v,
                                 int C, int T, double eps) {
    extern __shared__ double sm[];                      // [T/2][8]
    const int groups = lv.D / 8;
    const int g = blockIdx.x % groups;
    const int kv = (blockIdx.x / groups) & 1;
    const int bh = blockIdx.x / groups / 2;
    const int h = bh % lv.H, b = bh / lv.H;
    const float* x = kv ? v : k;
    const int t = threadIdx.x;                          // 0 .. T/2-1
    const int half = T / 2;
    const long long rs = (long long)lv.H * lv.D;
    const float* r0 = x + ((long long)b * C + t) * rs + (long long)h * lv.D + g * 8;
    const float* r1 = r0 + (long long)half * rs;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const double a0 = (double)r0[c], a1 = (double)r1[c];
        sm[t * 8 + c] = __dadd_rn(__dmul_rn(a0, a0), __dmul_rn(a1, a1));
    }
    __syncthreads();
    for (int stride = half / 2; stride >= 1; stride >>= 1) {
        if (t < stride) {
#pragma unroll
            for (int c = 0; c < 8; ++c) sm[t * 8 + c] = __dadd_rn(sm[t * 8 + c], sm[(t + stride) * 8 + c]);
        }
        __syncthreads();
    }
    if (t < 8) {
        const double mean = __dadd_rn(sm[t] / (double)T, eps);
        lv.scales[((long long)(b * lv.H + h) * 2 + kv) * lv.D + g * 8 + t] = __double2float_rn(sqrt(mean));
    }
}

}  // namespace

cudaError_t launch_append(const LayerView& lv, const float* k, const float* v, long long n, int C,
                          cudaStream_t st) {
    if (n + C > (1LL << 31) || lv.B > 65535 || 2LL * lv.H > 65535) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)((C + WARPS_PER_CTA - 1) / WARPS_PER_CTA), (unsigned)(2 * lv.H), (unsigned)lv.B);
    const dim3 block(32 * WARPS_PER_CTA);
    RingDiv rd{0, 0, 0};
    if (lv.W > 0) {
        uint32_t sh = 0;
        while ((1LL << sh) < lv.W) ++sh;
        rd.s = sh;
        rd.m = (unsigned long long)((((unsigned __int128)1 << (32 + sh)) + (unsigned)lv.W - 1) / (unsigned)lv.W);
        rd.n_mod_w = (uint32_t)(n % lv.W);
    }
    const uint32_t n32 = (uint32_t)n, C32 = (uint32_t)C;
    uint32_t done = 0;
    if (lv.kivi) {
        // per-channel K: quantize the groups this append completes (before the ring and the
        // pending rows are overwritten), then the append sends the rest to the pending rows
        const long long e0 = lv.W ? std::max(0LL, n - lv.W) : n;
        const long long e1 = lv.W ? std::max(0LL, n + C - lv.W) : n + C;
        const long long g0 = e0 / 32, g1 = e1 / 32;
        done = (uint32_t)(32 * g1);
        if (g1 > g0) {
            const long long ng = g1 - g0;
            const unsigned gg = (unsigned)(lv.B * lv.H * ng);
            const size_t smem = (size_t)32 * lv.D * sizeof(float);
            switch (lv.D / 32) {
                case 1: kivi_group_kernel<1><<<gg, 256, smem, st>>>(lv, k, n32, C32, (uint32_t)g0, (uint32_t)ng); break;
                case 2: kivi_group_kernel<2><<<gg, 256, smem, st>>>(lv, k, n32, C32, (uint32_t)g0, (uint32_t)ng); break;
                case 4: kivi_group_kernel<4><<<gg, 256, smem, st>>>(lv, k, n32, C32, (uint32_t)g0, (uint32_t)ng); break;
                case 8: kivi_group_kernel<8><<<gg, 256, smem, st>>>(lv, k, n32, C32, (uint32_t)g0, (uint32_t)ng); break;
                default: return cudaErrorInvalidValue;
            }
            cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
    }
    switch (lv.D / 32) {
        case 1: append_kernel<1><<<grid, block, 0, st>>>(lv, k, v, n32, C32, done, rd); break;
        case 2: append_kernel<2><<<grid, block, 0, st>>>(lv, k, v, n32, C32, done, rd); break;
        case 4: append_kernel<4><<<grid, block, 0, st>>>(lv, k, v, n32, C32, done, rd); break;
        case 8: append_kernel<8><<<grid, block, 0, st>>>(lv, k, v, n32, C32, done, rd); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_calibrate(const LayerView& lv, const float* k, const float* v, int C, int T,
                             double eps, cudaStream_t st) {
    const unsigned grid = (unsigned)(lv.B * lv.H * 2 * (lv.D / 8));
    const size_t smem = (size_t)(T / 2) * 8 * sizeof(double);
    calibrate_kernel<<<grid, T / 2, smem, st>>>(lv, k, v, C, T, eps);
    return cudaGetLastError();
}

}  // namespace kvq
