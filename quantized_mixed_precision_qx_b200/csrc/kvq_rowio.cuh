// kvq_rowio.cuh -- per-lane row access shared by the append and attention kernels.
//
// A warp reads or writes one row of D = 32*CPL channels; lane l owns channels
// [l*CPL, (l+1)*CPL). Row layout: see kvq_internal.cuh.
#pragma once
#include "kvq_internal.cuh"

namespace kvq {

template <int LPB>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
    for (int o = 1; o < LPB; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
template <int LPB>
__device__ __forceinline__ float group_min(float v) {
#pragma unroll
    for (int o = 1; o < LPB; o <<= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Load this lane's CPL floats of a float32 row.
template <int CPL>
__device__ __forceinline__ void load_row_f32(const float* __restrict__ row, int lane, float (&x)[CPL]) {
    const float* p = row + lane * CPL;
    if constexpr (CPL % 4 == 0) {
#pragma unroll
        for (int j = 0; j < CPL; j += 4) {
            float4 t = __ldcs(reinterpret_cast<const float4*>(p + j));
            x[j] = t.x; x[j + 1] = t.y; x[j + 2] = t.z; x[j + 3] = t.w;
        }
    } else if constexpr (CPL == 2) {
        float2 t = __ldcs(reinterpret_cast<const float2*>(p));
        x[0] = t.x; x[1] = t.y;
    } else {
        x[0] = __ldcs(p);
    }
}

// Read the CPL*w bits of a plane holding the codes of channels lane*CPL .. lane*CPL + CPL - 1
// of a row with nb blocks (CPL <= 8: they lie inside one 8-channel piece).
template <int CPL>
__device__ __forceinline__ uint64_t load_plane_bits(const uint8_t* plane, int nb, int lane, int w) {
    const int nbits = CPL * w;
    const int bit = plane_bit(nb, lane * CPL, w);
    const uint8_t* p = plane + (bit >> 3);
    switch (nbits) {
        case 64: return *reinterpret_cast<const unsigned long long*>(p);
        case 32: return *reinterpret_cast<const uint32_t*>(p);
        case 16: return *reinterpret_cast<const uint16_t*>(p);
        case 8: return *p;
        default: return (uint64_t)((*p >> (bit & 7)) & ((1u << nbits) - 1));
    }
}

// Write the CPL*w bits (value v) of channels lane*CPL .. lane*CPL + CPL - 1 into a plane of a
// row with nb blocks. Sub-byte pieces are gathered into whole bytes across lanes first (all
// lanes of the warp participate; the lanes sharing a byte are consecutive).
template <int CPL>
__device__ __forceinline__ void store_plane_bits(uint8_t* plane, int nb, int lane, int w, uint64_t v) {
    const int nbits = CPL * w;
    const int bit = plane_bit(nb, lane * CPL, w);
    uint8_t* p = plane + (bit >> 3);
    if (nbits >= 8) {
        switch (nbits) {
            case 64: *reinterpret_cast<unsigned long long*>(p) = v; break;
            case 32: *reinterpret_cast<uint32_t*>(p) = (uint32_t)v; break;
            case 16: *reinterpret_cast<uint16_t*>(p) = (uint16_t)v; break;
            default: *p = (uint8_t)v; break;
        }
        return;
    }
    uint32_t part = (uint32_t)v << (bit & 7);
    const int lanes_per_byte = 8 / nbits;
    for (int o = 1; o < lanes_per_byte; o <<= 1) part |= __shfl_xor_sync(0xffffffffu, part, o);
    if ((lane % lanes_per_byte) == 0) *p = (uint8_t)part;
}

// Dequantize this lane's CPL values of a stored row (exact in float32: d * integer).
template <int CPL>
__device__ __forceinline__ void load_row_values(const uint8_t* __restrict__ row, const RowFmt& f, int lane,
                                                float (&x)[CPL]) {
    if (f.kind != 0) {
        const uint16_t* h = reinterpret_cast<const uint16_t*>(row) + lane * CPL;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const uint16_t b = h[j];
            x[j] = (f.kind == 1) ? __uint_as_float((uint32_t)b << 16)
                                 : __half2float(__ushort_as_half(b));
        }
        return;
    }
    const int blk = (lane * CPL) >> 5;
    const float d = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(row)[blk]));
    const float m = f.asym ? __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(row + f.off_m)[blk])) : 0.f;
    const int nb = CPL;   // blocks per row: D / 32 = CPL
    const uint64_t p0 = load_plane_bits<CPL>(row + f.off_p0, nb, lane, f.w0);
    const uint64_t p1 = f.w1 ? load_plane_bits<CPL>(row + f.off_p1, nb, lane, f.w1) : 0;
    const uint32_t m0 = (1u << f.w0) - 1, m1 = (1u << f.w1) - 1;
    const int off = 1 << (f.bits - 1);
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const int u = (int)(((p0 >> (j * f.w0)) & m0) | (((p1 >> (j * f.w1)) & m1) << f.w0));
        x[j] = f.asym ? __fadd_rn(__fmul_rn(d, (float)u), m) : __fmul_rn(d, (float)(u - off));
    }
}

}  // namespace kvq
