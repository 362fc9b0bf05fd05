// kvq_mma.cuh -- register-level building blocks of the tensor-core decode kernel:
// m16n8k16 MMAs, TMA bulk copies with mbarriers (bounded waits), and the per-format
// unpacking of packed code planes straight into MMA A-fragments.
//
// Exactness: a qX code (offset removed) is a small integer and exact in fp16, so the
// A operand carries codes without rounding. The other operand (the query, or the
// softmax weight times the block scale) is split into fp16 hi + lo parts, so each
// product is carried to ~22 significant bits with fp32 accumulation. A 16-bit float
// ring row is exact in its own type; bf16 rows pair with a 3-way bf16 split.
#pragma once
#include "kvq_internal.cuh"

namespace kvq {
namespace mma {

// ---------------------------------------------------------------- formats
template <int F>
struct Fmt {
    static constexpr bool is_float = (F == F_BF16 || F == F_F16);
    static constexpr bool is_bf16 = (F == F_BF16);
    static constexpr int bits = is_float ? 16 : ((F / 2 == 5) ? 8 : 2 + F / 2);
    static constexpr bool asym = !is_float && (F & 1);
    static constexpr int w0 = is_float ? 16 : (bits == 8 ? 8 : (bits >= 4 ? 4 : 2));
    static constexpr int w1 = is_float ? 0 : bits - w0;
    static constexpr int off = asym ? 0 : (is_float ? 0 : (1 << (bits - 1)));
    // V codes enter the P V MMA centred: u - 2^(bits-1) (qX_0) or u - (2^bits - 1)/2 (qX_1, a
    // half-integer, exact in fp16 for these small codes; the min term then carries
    // m + d * (2^bits - 1)/2). With all-positive codes the MMA sum and the min term grow large
    // with opposite signs over long splits, and their cancellation magnifies the accumulation
    // error of the MMA.
    static constexpr float vcenter = is_float ? 0.f : (asym ? 0.5f * (float)((1 << bits) - 1) : (float)(1 << (bits - 1)));
    // row byte offsets for nb blocks (see kvq_internal.cuh)
    __device__ static constexpr int off_m(int nb) { return 2 * nb; }
    __device__ static constexpr int off_p0(int nb) { return is_float ? 0 : 2 * nb * (asym ? 2 : 1); }
    __device__ static constexpr int off_p1(int nb) { return off_p0(nb) + 32 * nb * w0 / 8; }
    // number of B-operand parts (split of the non-code operand)
    static constexpr int parts = is_bf16 ? 3 : 2;
    // bytes of one row of nb blocks and its 16-byte-padded stride (see kvq_internal.cuh)
    __host__ __device__ static constexpr int row_bytes(int nb) {
        return is_float ? 64 * nb : off_p0c(nb) + 4 * nb * (w0 + w1);
    }
    __host__ __device__ static constexpr int stride(int nb) { return (row_bytes(nb) + 15) & ~15; }
    __host__ __device__ static constexpr int off_p0c(int nb) { return is_float ? 0 : 2 * nb * (asym ? 2 : 1); }
};

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// (a & mask) | c  in one LOP3
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t mask, uint32_t c) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(c));
    return r;
}

template <int S>
__device__ __forceinline__ uint32_t shift(uint32_t x) {   // S > 0: left, S < 0: right
    if constexpr (S > 0) return x << S;
    else if constexpr (S < 0) return x >> (-S);
    else return x;
}

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int F>
__device__ __forceinline__ void mma_f(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (Fmt<F>::is_bf16) mma_bf16(c, a, b0, b1);
    else mma_f16(c, a, b0, b1);
}

// Exact fp16 -> fp32 without the conversion unit: the fp16 bit pattern shifted into the
// fp32 exponent/mantissa fields is the fp32 value x * 2^-112 (normal or subnormal fp16
// alike), so one exact multiply by 2^112 restores x. lo16 / hi16 select a half of w.
__device__ __forceinline__ float h2f_lo(uint32_t w) {
    const uint32_t u = ((w << 13) & 0x0FFFE000u) | ((w << 16) & 0x80000000u);
    return __uint_as_float(u) * 5.192296858534828e33f;   // 2^112
}
__device__ __forceinline__ float h2f_hi(uint32_t w) {
    const uint32_t u = ((w >> 3) & 0x0FFFE000u) | (w & 0x80000000u);
    return __uint_as_float(u) * 5.192296858534828e33f;
}

// 2^x on the special-function unit (relative error ~2^-22; inputs <= 0 or small)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Split x into `parts` values of the MMA's 16-bit type whose sum carries x to about
// 11 (fp16) or 8 (bf16) significant bits per part. The high part is x with its fp32
// mantissa truncated to the 16-bit type's width (exactly representable in range), the
// next part is the exact fp32 remainder, rounded; two values pack into one register.
template <int F>
__device__ __forceinline__ void split_pack(float x0, float x1, uint32_t (&out)[3]) {
    if constexpr (Fmt<F>::is_bf16) {
        const float h0 = __uint_as_float(__float_as_uint(x0) & 0xFFFF0000u);
        const float h1 = __uint_as_float(__float_as_uint(x1) & 0xFFFF0000u);
        const float r0 = x0 - h0, r1 = x1 - h1;
        const float m0 = __uint_as_float(__float_as_uint(r0) & 0xFFFF0000u);
        const float m1 = __uint_as_float(__float_as_uint(r1) & 0xFFFF0000u);
        out[0] = (__float_as_uint(h0) >> 16) | (__float_as_uint(h1) & 0xFFFF0000u);
        out[1] = (__float_as_uint(m0) >> 16) | (__float_as_uint(m1) & 0xFFFF0000u);
        __nv_bfloat162 l = __floats2bfloat162_rn(r0 - m0, r1 - m1);
        out[2] = *reinterpret_cast<uint32_t*>(&l);
    } else {
        const float h0 = __uint_as_float(__float_as_uint(x0) & 0xFFFFE000u);
        const float h1 = __uint_as_float(__float_as_uint(x1) & 0xFFFFE000u);
        __half2 h = __floats2half2_rn(h0, h1);
        __half2 l = __floats2half2_rn(x0 - h0, x1 - h1);
        out[0] = *reinterpret_cast<uint32_t*>(&h);
        out[1] = *reinterpret_cast<uint32_t*>(&l);
        out[2] = 0;
    }
}

// ---------------------------------------------------------------- mbarrier + bulk copy
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// order this thread's generic-proxy shared-memory writes before later async-proxy (TMA) writes
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// With `suspend`, a waiting thread may be suspended by the hardware for up to
// MBAR_SUSPEND_NS per try (it is woken when the phase completes), so waiting warps leave
// the issue slots to the others; without it the wait polls (lower wake-up latency).
constexpr uint32_t MBAR_SUSPEND_NS = 20000;
// Bounded wait for the phase with parity `parity` to complete. Returns false once about
// `limit_ns` nanoseconds have passed without completion (the caller records an error and
// stops waiting), so a wait that can never finish ends the kernel instead of hanging it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = 2000000000ull,
                                          bool suspend = true) {
    const uint32_t a = smem_u32(bar);
    uint64_t start = 0;
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        if (suspend) {
            asm volatile(
                "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
                : "=r"(done) : "r"(a), "r"(parity), "r"(MBAR_SUSPEND_NS) : "memory");
        } else {
            asm volatile(
                "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
                : "=r"(done) : "r"(a), "r"(parity) : "memory");
        }
        if (done) return true;
        if ((i & 63) == 0) {
            const uint64_t now = global_ns();
            if (i == 0) start = now;
            else if (now - start > limit_ns) return false;
        }
    }
}
// Non-blocking test of the phase with parity `parity` (true once it has completed).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return done != 0;
}
// 1-D bulk copy global -> shared (TMA engine), completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- fp16 magic
// 0x6400 is fp16 1024.0: OR-ing a code u < 1024 into the mantissa gives 1024 + u.
constexpr uint32_t MAGIC = 0x64006400u;

template <int F, int OFF = Fmt<F>::off>
__device__ __forceinline__ uint32_t debias(uint32_t x) {
    // (1024 + u) - (1024 + off) = u - off, exact
    constexpr uint32_t bias_h = 0x6400u + (uint32_t)OFF;   // fp16 bits of 1024 + off (exact, off < 1024)
    const __half2 b = __halves2half2(__ushort_as_half((unsigned short)bias_h), __ushort_as_half((unsigned short)bias_h));
    __half2 v = *reinterpret_cast<__half2*>(&x);
    __half2 r = __hsub2(v, b);
    return *reinterpret_cast<uint32_t*>(&r);
}

}  // namespace mma
}  // namespace kvq

namespace kvq {
namespace mma {

// ---------------------------------------------------------------- K side (QK^T)
// A operand of S^T = K Q^T for one 32-channel block b: rows are the sub-tile tokens
// (g, g + 8), the k dimension runs over channels. Thread t (lane & 3) holds channels
// 8t..8t+7 of the block; per MMA m in {0, 1} the k order is
//   quantized: (8t+2m, 8t+2m+4, 8t+2m+1, 8t+2m+5)   16-bit float: 8t+4m+{0,1,2,3}
// (q_channel gives the same order to the query operand).
template <int F>
__device__ __forceinline__ int q_channel(int t, int m, int slot) {
    if constexpr (Fmt<F>::is_float) return 8 * t + 4 * m + slot;
    else return 8 * t + 2 * m + ((slot & 1) ? 4 : 0) + (slot >> 1);
}

// four code pairs (n_j, n_{j+4}) of 8 consecutive channels of one row, biased by 1024
template <int F>
__device__ __forceinline__ void k_pairs(const uint8_t* row, int nb, int b, int t, uint32_t (&p)[4]) {
    using FT = Fmt<F>;
    constexpr int w0 = FT::w0, w1 = FT::w1;
    const uint8_t* p0 = row + FT::off_p0(nb);
    if constexpr (w0 == 4) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p0 + piece_off(nb, b, t, 4));
        p[0] = and_or(w, 0x000F000Fu, MAGIC);
        p[1] = and_or(w >> 4, 0x000F000Fu, MAGIC);
        p[2] = and_or(w >> 8, 0x000F000Fu, MAGIC);
        p[3] = and_or(w >> 12, 0x000F000Fu, MAGIC);
    } else if constexpr (w0 == 8) {
        const uint2 w = *reinterpret_cast<const uint2*>(p0 + piece_off(nb, b, t, 8));
#pragma unroll
        for (int j = 0; j < 4; ++j) p[j] = and_or(prmt(w.x, w.y, (uint32_t)(j | ((4 + j) << 8))), 0x00FF00FFu, MAGIC);
    } else {  // w0 == 2
        const uint32_t hw = *reinterpret_cast<const uint16_t*>(p0 + piece_off(nb, b, t, 2));
        const uint32_t x = prmt(hw, 0u, 0x4140u);
        p[0] = and_or(x, 0x00030003u, MAGIC);
        p[1] = and_or(x >> 2, 0x00030003u, MAGIC);
        p[2] = and_or(x >> 4, 0x00030003u, MAGIC);
        p[3] = and_or(x >> 6, 0x00030003u, MAGIC);
    }
    if constexpr (w1 == 2) {
        const uint8_t* p1 = row + FT::off_p1(nb);
        const uint32_t hw = *reinterpret_cast<const uint16_t*>(p1 + piece_off(nb, b, t, 2));
        const uint32_t x = prmt(hw, 0u, 0x4140u);
        constexpr uint32_t M = 0x00030003u << w0;
        p[0] = and_or(shift<w0 - 0>(x), M, p[0]);
        p[1] = and_or(shift<w0 - 2>(x), M, p[1]);
        p[2] = and_or(shift<w0 - 4>(x), M, p[2]);
        p[3] = and_or(shift<w0 - 6>(x), M, p[3]);
    } else if constexpr (w1 == 1) {
        const uint8_t* p1 = row + FT::off_p1(nb);
        const uint32_t by = p1[piece_off(nb, b, t, 1)];
        const uint32_t x = by | (by << 12);
        constexpr uint32_t M = 0x00010001u << w0;
        p[0] = and_or(shift<w0 - 0>(x), M, p[0]);
        p[1] = and_or(shift<w0 - 1>(x), M, p[1]);
        p[2] = and_or(shift<w0 - 2>(x), M, p[2]);
        p[3] = and_or(shift<w0 - 3>(x), M, p[3]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) p[j] = debias<F>(p[j]);
}

template <int F>
__device__ __forceinline__ void k_frags(const uint8_t* rg, const uint8_t* rg8, int nb, int b, int t,
                                        uint32_t (&a)[2][4]) {
    if constexpr (Fmt<F>::is_float) {
        const uint4 x = *reinterpret_cast<const uint4*>(rg + 64 * b + 16 * t);
        const uint4 y = *reinterpret_cast<const uint4*>(rg8 + 64 * b + 16 * t);
        a[0][0] = x.x; a[0][1] = y.x; a[0][2] = x.y; a[0][3] = y.y;
        a[1][0] = x.z; a[1][1] = y.z; a[1][2] = x.w; a[1][3] = y.w;
    } else {
        uint32_t pg[4], pg8[4];
        k_pairs<F>(rg, nb, b, t, pg);
        k_pairs<F>(rg8, nb, b, t, pg8);
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            a[m][0] = pg[2 * m];
            a[m][1] = pg8[2 * m];
            a[m][2] = pg[2 * m + 1];
            a[m][3] = pg8[2 * m + 1];
        }
    }
}

// ---------------------------------------------------------------- V side (P V)
// A operand of O^T = V^T P^T for block b: rows are channels, the k dimension runs over
// the sub-tile tokens (2t, 2t+1, 2t+8, 2t+9) held by thread (g, t). Thread g covers
// channels 8k + 4hs + i (k = g >> 1, hs = g & 1, i = 0..3); in M-tile mt row g is
// channel 8k + 4hs + 2mt and row g + 8 is channel 8k + 4hs + 2mt + 1.
__device__ __forceinline__ int v_channel(int g, int mt, int row_hi) {
    return 8 * (g >> 1) + 4 * (g & 1) + 2 * mt + row_hi;
}

// four channel pairs over two tokens (ra, rb): pair i = (token a, token b) of channel
// 8k + 4hs + i, biased by 1024 (quantized) or raw 16-bit values (float formats)
template <int F>
__device__ __forceinline__ void v_pairs(const uint8_t* ra, const uint8_t* rb, int nb, int b, int g,
                                        uint32_t (&p)[4]) {
    using FT = Fmt<F>;
    constexpr int w0 = FT::w0, w1 = FT::w1;
    const int k = g >> 1, hs = g & 1;
    if constexpr (FT::is_float) {
        const uint2 wa = *reinterpret_cast<const uint2*>(ra + 64 * b + 16 * k + 8 * hs);
        const uint2 wb = *reinterpret_cast<const uint2*>(rb + 64 * b + 16 * k + 8 * hs);
        p[0] = prmt(wa.x, wb.x, 0x5410u);
        p[1] = prmt(wa.x, wb.x, 0x7632u);
        p[2] = prmt(wa.y, wb.y, 0x5410u);
        p[3] = prmt(wa.y, wb.y, 0x7632u);
        return;
    } else {
        const int o0 = FT::off_p0(nb);
        if constexpr (w0 == 4) {
            const uint32_t wa = *reinterpret_cast<const uint32_t*>(ra + o0 + piece_off(nb, b, k, 4));
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(rb + o0 + piece_off(nb, b, k, 4));
            const uint32_t x = prmt(wa, wb, hs ? 0x7632u : 0x5410u);
            p[0] = and_or(x, 0x000F000Fu, MAGIC);
            p[1] = and_or(x >> 4, 0x000F000Fu, MAGIC);
            p[2] = and_or(x >> 8, 0x000F000Fu, MAGIC);
            p[3] = and_or(x >> 12, 0x000F000Fu, MAGIC);
        } else if constexpr (w0 == 8) {
            const uint32_t wa = *reinterpret_cast<const uint32_t*>(ra + o0 + piece_off(nb, b, k, 8) + 4 * hs);
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(rb + o0 + piece_off(nb, b, k, 8) + 4 * hs);
#pragma unroll
            for (int i = 0; i < 4; ++i) p[i] = and_or(prmt(wa, wb, (uint32_t)(i | ((4 + i) << 8))), 0x00FF00FFu, MAGIC);
        } else {  // w0 == 2
            const uint32_t ba = ra[o0 + piece_off(nb, b, k, 2) + hs];
            const uint32_t bb = rb[o0 + piece_off(nb, b, k, 2) + hs];
            const uint32_t x = prmt(ba, bb, 0x5410u);
            p[0] = and_or(x, 0x00030003u, MAGIC);
            p[1] = and_or(x >> 2, 0x00030003u, MAGIC);
            p[2] = and_or(x >> 4, 0x00030003u, MAGIC);
            p[3] = and_or(x >> 6, 0x00030003u, MAGIC);
        }
        if constexpr (w1 == 2) {
            const int o1 = FT::off_p1(nb);
            const uint32_t ha = ra[o1 + piece_off(nb, b, k, 2) + hs];
            const uint32_t hb = rb[o1 + piece_off(nb, b, k, 2) + hs];
            const uint32_t y = prmt(ha, hb, 0x5410u);
            constexpr uint32_t M = 0x00030003u << w0;
            p[0] = and_or(shift<w0 - 0>(y), M, p[0]);
            p[1] = and_or(shift<w0 - 2>(y), M, p[1]);
            p[2] = and_or(shift<w0 - 4>(y), M, p[2]);
            p[3] = and_or(shift<w0 - 6>(y), M, p[3]);
        } else if constexpr (w1 == 1) {
            const int o1 = FT::off_p1(nb);
            const uint32_t ha = ra[o1 + piece_off(nb, b, k, 1)];
            const uint32_t hb = rb[o1 + piece_off(nb, b, k, 1)];
            const uint32_t y = prmt(ha, hb, 0x5410u) >> (4 * hs);
            constexpr uint32_t M = 0x00010001u << w0;
            p[0] = and_or(shift<w0 - 0>(y), M, p[0]);
            p[1] = and_or(shift<w0 - 1>(y), M, p[1]);
            p[2] = and_or(shift<w0 - 2>(y), M, p[2]);
            p[3] = and_or(shift<w0 - 3>(y), M, p[3]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (FT::asym) {
                // (1024 + u) - 1024 = u, then u - c: both exact in fp16
                const __half2 u2 = *reinterpret_cast<const __half2*>(&p[i]);
                const __half2 r = __hsub2(__hsub2(u2, __float2half2_rn(1024.f)), __float2half2_rn(FT::vcenter));
                p[i] = *reinterpret_cast<const uint32_t*>(&r);
            } else {
                p[i] = debias<F>(p[i]);
            }
        }
    }
}

// tokens r0..r3 = sub-tile rows 2t, 2t+1, 2t+8, 2t+9 (rows past the data hold finite
// stale values; their P entries are zero)
template <int F>
__device__ __forceinline__ void v_frags(const uint8_t* r0, const uint8_t* r1, const uint8_t* r2, const uint8_t* r3,
                                        int nb, int b, int g, uint32_t (&a)[2][4]) {
    uint32_t pa[4], pb[4];
    v_pairs<F>(r0, r1, nb, b, g, pa);
    v_pairs<F>(r2, r3, nb, b, g, pb);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        a[mt][0] = pa[2 * mt];
        a[mt][1] = pa[2 * mt + 1];
        a[mt][2] = pb[2 * mt];
        a[mt][3] = pb[2 * mt + 1];
    }
}

// Quantized V with the block scale folded into the A operand: for the token pairs
// (r0, r1) and (r2, r3), x = d * (u - off) is computed in fp16 as hi = RN(d * c) and the
// exact remainder lo = d * c - hi (fused multiply-add, single rounding; d * c has at most
// 17 significant bits, so hi + lo == d * c unless the fp16 subnormal range is reached).
// vmul: a power of two 2^-e in both fp16 halves, applied to the scales first (exact while
// d * 2^-e stays representable) so that every d * c of the cache fits fp16; the caller
// multiplies the accumulated output by 2^e.
template <int F>
__device__ __forceinline__ void v_frags_scaled(const uint8_t* r0, const uint8_t* r1, const uint8_t* r2,
                                               const uint8_t* r3, int nb, int b, int g, uint32_t vmul,
                                               uint32_t (&ahi)[2][4], uint32_t (&alo)[2][4]) {
    uint32_t pa[4], pb[4];
    v_pairs<F>(r0, r1, nb, b, g, pa);
    v_pairs<F>(r2, r3, nb, b, g, pb);
    const uint32_t d01 = prmt(reinterpret_cast<const uint16_t*>(r0)[b], reinterpret_cast<const uint16_t*>(r1)[b], 0x5410u);
    const uint32_t d23 = prmt(reinterpret_cast<const uint16_t*>(r2)[b], reinterpret_cast<const uint16_t*>(r3)[b], 0x5410u);
    const __half2 vm = *reinterpret_cast<const __half2*>(&vmul);
    const __half2 da = __hmul2_rn(*reinterpret_cast<const __half2*>(&d01), vm);
    const __half2 db = __hmul2_rn(*reinterpret_cast<const __half2*>(&d23), vm);
    uint32_t ha[4], la[4], hb[4], lb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 xa = *reinterpret_cast<const __half2*>(&pa[i]);
        const __half2 xb = *reinterpret_cast<const __half2*>(&pb[i]);
        const __half2 h1 = __hmul2_rn(xa, da);
        const __half2 h2 = __hmul2_rn(xb, db);
        const __half2 l1 = __hfma2(xa, da, __hneg2(h1));
        const __half2 l2 = __hfma2(xb, db, __hneg2(h2));
        ha[i] = *reinterpret_cast<const uint32_t*>(&h1);
        hb[i] = *reinterpret_cast<const uint32_t*>(&h2);
        la[i] = *reinterpret_cast<const uint32_t*>(&l1);
        lb[i] = *reinterpret_cast<const uint32_t*>(&l2);
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        ahi[mt][0] = ha[2 * mt]; ahi[mt][1] = ha[2 * mt + 1]; ahi[mt][2] = hb[2 * mt]; ahi[mt][3] = hb[2 * mt + 1];
        alo[mt][0] = la[2 * mt]; alo[mt][1] = la[2 * mt + 1]; alo[mt][2] = lb[2 * mt]; alo[mt][3] = lb[2 * mt + 1];
    }
}

// ---------------------------------------------------------------- wide loads of pieces
// BYTES bytes at p (a multiple of ALIGN, the guaranteed alignment of p) into 32-bit words
// (BYTES < 4: the low bytes of w[0]).
template <int BYTES, int ALIGN>
__device__ __forceinline__ void load_bytes(const uint8_t* p, uint32_t (&w)[(BYTES + 3) / 4]) {
    if constexpr (BYTES >= 16 && ALIGN >= 16) {
#pragma unroll
        for (int i = 0; i < BYTES / 16; ++i) {
            const uint4 v = reinterpret_cast<const uint4*>(p)[i];
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else if constexpr (BYTES >= 8 && ALIGN >= 8) {
#pragma unroll
        for (int i = 0; i < BYTES / 8; ++i) {
            const uint2 v = reinterpret_cast<const uint2*>(p)[i];
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else if constexpr (BYTES >= 4) {
#pragma unroll
        for (int i = 0; i < BYTES / 4; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
    } else if constexpr (BYTES == 2) {
        w[0] = *reinterpret_cast<const uint16_t*>(p);
    } else {
        w[0] = *p;
    }
}

// The pieces of slot t of blocks b0 .. b0 + HB - 1 of one stored row (plane 0, plane 1, the
// block scales and, for qX_1, the mins), loaded with the widest aligned loads: slot t of
// consecutive blocks is contiguous in each plane.
template <int F, int NB, int HB>
struct RowPieces {
    using FT = Fmt<F>;
    static constexpr int B0 = HB * FT::w0, B1 = HB * FT::w1;
    uint32_t p0[(B0 + 3) / 4];
    uint32_t p1[B1 > 0 ? (B1 + 3) / 4 : 1];
    uint32_t d[(2 * HB + 3) / 4];
    uint32_t m[FT::asym ? (2 * HB + 3) / 4 : 1];
    // alignment of a run of `len` bytes (a power of two) at a multiple of len past offset off
    // of a 16-byte-aligned row
    static constexpr int run_align(int off, int len) {
        const int a = (off % 16 == 0) ? 16 : (off % 8 == 0) ? 8 : (off % 4 == 0) ? 4 : (off % 2 == 0) ? 2 : 1;
        const int l = len >= 16 ? 16 : len;
        return a < l ? a : l;
    }

    // row: a 16-byte-aligned stored row; b0 = HB * (0 or 1), so each run starts at a multiple
    // of its own length inside its plane
    __device__ __forceinline__ void load(const uint8_t* row, int b0, int t) {
        constexpr int o0 = FT::off_p0c(NB), o1 = o0 + 4 * NB * FT::w0;
        load_bytes<B0, run_align(o0, B0)>(row + o0 + piece_off(NB, b0, t, FT::w0), p0);
        if constexpr (B1 > 0) load_bytes<B1, run_align(o1, B1)>(row + o1 + piece_off(NB, b0, t, FT::w1), p1);
        load_bytes<2 * HB, run_align(0, 2 * HB)>(row + 2 * b0, d);
        if constexpr (FT::asym) load_bytes<2 * HB, run_align(2 * NB, 2 * HB)>(row + 2 * NB + 2 * b0, m);
    }
    // plane bytes of block j (0 <= j < HB) of this run
    __device__ __forceinline__ uint32_t w0word(int j) const {   // w0 == 4: the piece's 32 bits
        return p0[j];
    }
    __device__ __forceinline__ uint32_t half16(const uint32_t* w, int j) const {   // 2-byte piece j
        return (w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu;
    }
    __device__ __forceinline__ uint32_t byte8(const uint32_t* w, int j) const {    // 1-byte piece j
        return (w[j >> 2] >> (8 * (j & 3))) & 0xFFu;
    }
    __device__ __forceinline__ uint32_t dbits(int j) const { return (d[j >> 1] >> (16 * (j & 1))) & 0xFFFFu; }
    __device__ __forceinline__ uint32_t mbits(int j) const { return (m[j >> 1] >> (16 * (j & 1))) & 0xFFFFu; }
};

// K side: the four code pairs (n_j, n_{j+4}) of block j's piece, biased by 1024 (as k_pairs)
template <int F, int NB, int HB>
__device__ __forceinline__ void k_pairs_r(const RowPieces<F, NB, HB>& r, int j, uint32_t (&p)[4]) {
    using FT = Fmt<F>;
    constexpr int w0 = FT::w0, w1 = FT::w1;
    if constexpr (w0 == 4) {
        const uint32_t w = r.p0[j];
        p[0] = and_or(w, 0x000F000Fu, MAGIC);
        p[1] = and_or(w >> 4, 0x000F000Fu, MAGIC);
        p[2] = and_or(w >> 8, 0x000F000Fu, MAGIC);
        p[3] = and_or(w >> 12, 0x000F000Fu, MAGIC);
    } else if constexpr (w0 == 8) {
        const uint32_t wx = r.p0[2 * j], wy = r.p0[2 * j + 1];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = and_or(prmt(wx, wy, (uint32_t)(i | ((4 + i) << 8))), 0x00FF00FFu, MAGIC);
    } else {  // w0 == 2: a 2-byte piece, its bytes spread to the two halves
        const uint32_t x = prmt(r.p0[j >> 1], 0u, (j & 1) ? 0x4342u : 0x4140u);
        p[0] = and_or(x, 0x00030003u, MAGIC);
        p[1] = and_or(x >> 2, 0x00030003u, MAGIC);
        p[2] = and_or(x >> 4, 0x00030003u, MAGIC);
        p[3] = and_or(x >> 6, 0x00030003u, MAGIC);
    }
    if constexpr (w1 == 2) {
        const uint32_t x = prmt(r.p1[j >> 1], 0u, (j & 1) ? 0x4342u : 0x4140u);
        constexpr uint32_t M = 0x00030003u << w0;
        p[0] = and_or(shift<w0 - 0>(x), M, p[0]);
        p[1] = and_or(shift<w0 - 2>(x), M, p[1]);
        p[2] = and_or(shift<w0 - 4>(x), M, p[2]);
        p[3] = and_or(shift<w0 - 6>(x), M, p[3]);
    } else if constexpr (w1 == 1) {
        const uint32_t by = (r.p1[j >> 2] >> (8 * (j & 3))) & 0xFFu;
        const uint32_t x = by * 4097u;                 // by | by << 12 (no carries: by < 256)
        constexpr uint32_t M = 0x00010001u << w0;
        p[0] = and_or(shift<w0 - 0>(x), M, p[0]);
        p[1] = and_or(shift<w0 - 1>(x), M, p[1]);
        p[2] = and_or(shift<w0 - 2>(x), M, p[2]);
        p[3] = and_or(shift<w0 - 3>(x), M, p[3]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = debias<F>(p[i]);
}

// V side: the four channel pairs over two tokens (ra, rb) of block j, half hs of slot k's
// piece (channels 4 hs .. 4 hs + 3 of it), biased by 1024 and debiased / centred as v_pairs
template <int F, int NB, int HB>
__device__ __forceinline__ void v_pairs_r(const RowPieces<F, NB, HB>& ra, const RowPieces<F, NB, HB>& rb, int j,
                                          int hs, uint32_t (&p)[4]) {
    using FT = Fmt<F>;
    constexpr int w0 = FT::w0, w1 = FT::w1;
    if constexpr (w0 == 4) {
        const uint32_t x = prmt(ra.p0[j], rb.p0[j], hs ? 0x7632u : 0x5410u);
        p[0] = and_or(x, 0x000F000Fu, MAGIC);
        p[1] = and_or(x >> 4, 0x000F000Fu, MAGIC);
        p[2] = and_or(x >> 8, 0x000F000Fu, MAGIC);
        p[3] = and_or(x >> 12, 0x000F000Fu, MAGIC);
    } else if constexpr (w0 == 8) {
        const uint32_t wa = ra.p0[2 * j + hs], wb = rb.p0[2 * j + hs];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = and_or(prmt(wa, wb, (uint32_t)(i | ((4 + i) << 8))), 0x00FF00FFu, MAGIC);
    } else {  // w0 == 2: byte hs of the 2-byte piece of each row
        const int bsel = 2 * (j & 1) + hs;
        const uint32_t x = prmt(ra.p0[j >> 1], rb.p0[j >> 1], (uint32_t)(bsel | ((4 + bsel) << 8)));
        p[0] = and_or(x, 0x00030003u, MAGIC);
        p[1] = and_or(x >> 2, 0x00030003u, MAGIC);
        p[2] = and_or(x >> 4, 0x00030003u, MAGIC);
        p[3] = and_or(x >> 6, 0x00030003u, MAGIC);
    }
    if constexpr (w1 == 2) {
        const int bsel = 2 * (j & 1) + hs;
        const uint32_t y = prmt(ra.p1[j >> 1], rb.p1[j >> 1], (uint32_t)(bsel | ((4 + bsel) << 8)));
        constexpr uint32_t M = 0x00030003u << w0;
        p[0] = and_or(shift<w0 - 0>(y), M, p[0]);
        p[1] = and_or(shift<w0 - 2>(y), M, p[1]);
        p[2] = and_or(shift<w0 - 4>(y), M, p[2]);
        p[3] = and_or(shift<w0 - 6>(y), M, p[3]);
    } else if constexpr (w1 == 1) {
        const int bsel = j & 3;
        const uint32_t y = prmt(ra.p1[j >> 2], rb.p1[j >> 2], (uint32_t)(bsel | ((4 + bsel) << 8))) >> (4 * hs);
        constexpr uint32_t M = 0x00010001u << w0;
        p[0] = and_or(shift<w0 - 0>(y), M, p[0]);
        p[1] = and_or(shift<w0 - 1>(y), M, p[1]);
        p[2] = and_or(shift<w0 - 2>(y), M, p[2]);
        p[3] = and_or(shift<w0 - 3>(y), M, p[3]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (FT::asym) {
            const __half2 u2 = *reinterpret_cast<const __half2*>(&p[i]);
            const __half2 r = __hsub2(__hsub2(u2, __float2half2_rn(1024.f)), __float2half2_rn(FT::vcenter));
            p[i] = *reinterpret_cast<const uint32_t*>(&r);
        } else {
            p[i] = debias<F>(p[i]);
        }
    }
}

// A operand of O^T = V^T P^T for block j with the block scales (times vmul) folded in as an
// exact fp16 hi + lo pair, from the pieces of the four rows 2t, 2t+1, 2t+8, 2t+9
template <int F, int NB, int HB>
__device__ __forceinline__ void v_frags_scaled_r(const RowPieces<F, NB, HB>& r0, const RowPieces<F, NB, HB>& r1,
                                                 const RowPieces<F, NB, HB>& r2, const RowPieces<F, NB, HB>& r3,
                                                 int j, int hs, uint32_t vmul, uint32_t (&ahi)[2][4],
                                                 uint32_t (&alo)[2][4]) {
    uint32_t pa[4], pb[4];
    v_pairs_r<F, NB, HB>(r0, r1, j, hs, pa);
    v_pairs_r<F, NB, HB>(r2, r3, j, hs, pb);
    const uint32_t dsel = (j & 1) ? 0x7632u : 0x5410u;
    const uint32_t d01 = prmt(r0.d[j >> 1], r1.d[j >> 1], dsel);
    const uint32_t d23 = prmt(r2.d[j >> 1], r3.d[j >> 1], dsel);
    const __half2 vm = *reinterpret_cast<const __half2*>(&vmul);
    const __half2 da = __hmul2_rn(*reinterpret_cast<const __half2*>(&d01), vm);
    const __half2 db = __hmul2_rn(*reinterpret_cast<const __half2*>(&d23), vm);
    uint32_t ha[4], la[4], hb[4], lb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 xa = *reinterpret_cast<const __half2*>(&pa[i]);
        const __half2 xb = *reinterpret_cast<const __half2*>(&pb[i]);
        const __half2 h1 = __hmul2_rn(xa, da);
        const __half2 h2 = __hmul2_rn(xb, db);
        const __half2 l1 = __hfma2(xa, da, __hneg2(h1));
        const __half2 l2 = __hfma2(xb, db, __hneg2(h2));
        ha[i] = *reinterpret_cast<const uint32_t*>(&h1);
        hb[i] = *reinterpret_cast<const uint32_t*>(&h2);
        la[i] = *reinterpret_cast<const uint32_t*>(&l1);
        lb[i] = *reinterpret_cast<const uint32_t*>(&l2);
    }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
        ahi[mt][0] = ha[2 * mt]; ahi[mt][1] = ha[2 * mt + 1]; ahi[mt][2] = hb[2 * mt]; ahi[mt][3] = hb[2 * mt + 1];
        alo[mt][0] = la[2 * mt]; alo[mt][1] = la[2 * mt + 1]; alo[mt][2] = lb[2 * mt]; alo[mt][3] = lb[2 * mt + 1];
    }
}

}  // namespace mma
}  // namespace kvq
