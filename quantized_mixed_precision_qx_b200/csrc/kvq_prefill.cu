// kvq_prefill.cu -- causal chunked-prefill attention on 5th-generation tensor cores.
//
// The chunk's C rows were just appended at positions n - C .. n - 1; chunk row i attends
// to positions t <= n - C + i of the post-append cache (low-bit rows below the window,
// ring rows inside it). QK^T and PV are dense contractions, so they run as tcgen05 MMAs
// with fp32 accumulators in tensor memory. Two kernels:
//   - prefill_staged (below, with prefill_tiles): a head with more than one 128-row M-tile;
//     each K~ / V~ tile is dequantized once per head into a workspace image that every M-tile
//     CTA of the head streams;
//   - prefill_tc5 (this part): one M-tile per head (short chunks); each CTA dequantizes its
//     own tiles.
// Either kernel may split each M-tile's key range over several CTAs (partial O with the
// row's running max and sum) when that fills the GPU better; prefill_merge combines them.
//
// prefill_tc5:
//   CTA   = 128 query rows of one (batch, kv head): row r = chunk row * G + head in group,
//           TMEM lane r. 16 warps in three roles that signal each other through mbarriers:
//           warps 0-3 own one row per thread (softmax, epilogue), warps 4-14 dequantize,
//           lane 0 of warp 15 issues the MMAs and the bulk copies.
//   tile  = 32 key positions. Each tile is dequantized into shared memory as exact fp16
//           hi + lo parts (K~ = hi + lo; the query and P are split the same way), and
//           S = Qh Kh^T + Qh Kl^T + Ql Kh^T (3 passes, M128 N32 K16 steps) -> TMEM cols [0, 128)
//               (two partial sums over the channel halves, added by the softmax warps)
//               (double-buffered: the softmax reads S(t) while S(t + 1) is written)
//           O += Ph Vh + Ph Vl + Pl Vh    (3 passes, M128 N=D K16 steps) -> TMEM cols [256, 256 + D)
//   The softmax is row-local (each thread owns its row), with a lazily raised running max.
//   K~ (one or two tiles) and V~^T have buffers of their own, so the dequantization of one
//   tile overlaps the MMAs and the softmax of the previous one; the raw rows of tile t + 2
//   are fetched by bulk copies into a staging buffer as soon as tile t is dequantized.
//
// Shared memory of prefill_tc5 (head_dim D = 32 NB): Q hi 128 x D x 2 B (Q lo lives in TMEM), K~ hi/lo
// 2 x 32 x D x 2 B per K~ tile (K-major, 128-byte swizzle), V~^T hi/lo 2 x D x 32 x 2 B and
// P hi/lo 2 x 128 x 32 x 2 B (K-major, 64-byte swizzle), 2 staging buffers of 2 x 32 raw rows
// (sized by the widest row format).
#include <algorithm>

#include "kvq_internal.cuh"
#include "kvq_mma.cuh"
#include "kvq_tc5.cuh"

namespace kvq {
namespace {

constexpr int PM = 128;           // query rows per CTA
constexpr int PN = 32;            // key positions per tile
constexpr int PTHREADS = 512;     // 16 warps: 4 own the 128 TMEM rows, 11 dequantize, 1 issues
constexpr float PF_RESCALE = 8.0f;
// Tiles accumulated into O in tensor memory before the owners fold O into the output row
// with IEEE fp32 adds and the next P V~ starts a fresh accumulation: long accumulation runs
// in tensor memory lose precision (over 100k positions the error grows past 1e-4).
constexpr int PF_FOLD = 128;
constexpr int PF_MAX_SPLITS = 4;   // key-range splits of a staged prefill M-tile
constexpr int PF_OTF_MAX_SPLITS = 64;   // of an on-the-fly prefill M-tile (few rows, one wave)

struct PrefillArgs {
    LayerView lv;
    const float* q;               // [B][C][Hq][D]
    float* out;                   // [B][C][Hq][D]
    float qscale;                 // scale * log2(e)
    long long n;                  // cached positions (after the append)
    int C;                        // chunk rows
    int stage_half;               // bytes of one staging half (PN rows of the widest K|V row), multiple of 16
    int kbufs;                    // K~ buffers (2 when shared memory allows, else 1)
    int splits;                   // key-range splits per M-tile (1: rows finished in place)
    float* part;                  // splits > 1: [splits][B * C * Hq][D] unnormalised O, then
                                  // [splits][B * C * Hq][2] (running max, row sum)
};

// shared memory: Q hi, kbufs K~ tiles, V~^T, P (all 1024-byte multiples), then the 2
// staging buffers of 2 halves (raw K rows, raw V rows of one tile) and the barriers
__host__ __device__ constexpr size_t pf_tiles(int D, int kbufs) {
    return (size_t)PM * D * 2 /* Q hi */ + (size_t)kbufs * 2 * PN * D * 2 /* K~ hi, lo */ +
           2 * (size_t)D * PN * 2 /* V~^T hi, lo */ + 2 * (size_t)PM * PN * 2 /* P hi, lo */;
}
__host__ __device__ constexpr size_t pf_smem(int D, int kbufs, size_t stage_half) {
    return 1024 /* alignment slack */ + pf_tiles(D, kbufs) + 4 * stage_half + 256 /* barriers */ +
           1024 /* tail pad: no operand read can pass the end of the allocation */;
}

// split fp32 -> fp16 hi (truncated to 11 significant bits) + fp16 lo (rounded remainder)
__device__ __forceinline__ void split16(float x, __half& hi, __half& lo) {
    const float h = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
    hi = __float2half_rn(h);
    lo = __float2half_rn(x - h);
}

// 8 consecutive k-values of one operand row -> 16-byte chunks of the hi and lo tiles
__device__ __forceinline__ void store_chunk(uint8_t* hi_tile, uint8_t* lo_tile, int row, int k0, int rows,
                                           const float (&x)[8]) {
    __align__(16) __half h[8], l[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) split16(x[j], h[j], l[j]);
    const uint32_t off = t5::sw128_offset(row, k0, rows);
    *reinterpret_cast<uint4*>(hi_tile + off) = *reinterpret_cast<const uint4*>(h);
    *reinterpret_cast<uint4*>(lo_tile + off) = *reinterpret_cast<const uint4*>(l);
}

// same for a K-major tile with 64-byte rows (K extent 32)
__device__ __forceinline__ void store_chunk64(uint8_t* hi_tile, uint8_t* lo_tile, int row, int k0, const float (&x)[8]) {
    __align__(16) __half h[8], l[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) split16(x[j], h[j], l[j]);
    const uint32_t off = t5::sw64_offset(row, k0);
    *reinterpret_cast<uint4*>(hi_tile + off) = *reinterpret_cast<const uint4*>(h);
    *reinterpret_cast<uint4*>(lo_tile + off) = *reinterpret_cast<const uint4*>(l);
}

// Per-kernel copy (registers) of what the dequantization needs; built from the launch
// parameters once, so no field is ever read through a pointer into the parameter block.
struct SideView {
    const uint8_t* main;          // region of this (b, h)
    const uint8_t* ring;
    const float* scales;          // KVarN scales of this (b, h), or null
    RowFmt fmain, ftail;
    int W;
};

__device__ __forceinline__ SideView side_view(const LayerView& lv, int b, int h, int kv) {
    SideView v;
    v.main = lv.main[kv] + (long long)(b * lv.H + h) * lv.main_region[kv];
    v.ring = lv.W ? lv.ring[kv] + (long long)(b * lv.H + h) * lv.ring_region : nullptr;
    v.scales = lv.kvarn ? lv.scales + ((long long)(b * lv.H + h) * 2 + kv) * lv.D : nullptr;
    v.fmain = lv.fmt[kv];
    v.ftail = lv.tail;
    v.W = lv.W;
    return v;
}

// Raw words of channels c0..c0+7 of one stored row, fetched with loads that do not depend
// on each other (so a thread can have many rows in flight) and decoded afterwards.
struct Raw8 {
    uint64_t w;        // 8-byte-aligned window holding plane 0 (low-bit) / channels c0..c0+3 (16-bit)
    uint64_t w2;       // channels c0+4..c0+7 (16-bit rows only)
    uint32_t p1;       // 2-byte window holding plane 1
    uint32_t dm;       // d (low 16 bits), m (high 16 bits)
    uint32_t sh0, sh1; // bit offsets of the fields inside w / p1
    uint32_t sel;      // 0 = low-bit main row, 1 = tail row
};

// same, for a row already located (e.g. in the staging buffer) with its format
__device__ __forceinline__ void fetch8_row(const uint8_t* row, const RowFmt f, uint32_t sel, int c0, int nb,
                                           Raw8& r) {
    r.sel = sel;
    if (f.kind != 0) {
        const uint8_t* a = row + 2 * c0;                       // 16-byte aligned
        r.w = *reinterpret_cast<const unsigned long long*>(a);
        r.w2 = *reinterpret_cast<const unsigned long long*>(a + 8);
        r.p1 = 0; r.dm = 0; r.sh0 = 0; r.sh1 = 0;
        return;
    }
    const int blk = c0 >> 5;
    const uint32_t d = reinterpret_cast<const uint16_t*>(row)[blk];
    const uint32_t m = f.asym ? reinterpret_cast<const uint16_t*>(row + f.off_m)[blk] : 0u;
    r.dm = d | (m << 16);
    // the 8 channels c0 .. c0 + 7 form one piece of each plane (c0 is a multiple of 8)
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(row + f.off_p0 + piece_off(nb, blk, (c0 >> 3) & 3, f.w0));
    r.w = *reinterpret_cast<const unsigned long long*>(a0 & ~(uintptr_t)7);
    r.sh0 = (uint32_t)(a0 & 7) * 8;
    r.w2 = 0;
    if (f.w1) {
        const uintptr_t a1 = reinterpret_cast<uintptr_t>(row + f.off_p1 + piece_off(nb, blk, (c0 >> 3) & 3, f.w1));
        r.p1 = *reinterpret_cast<const uint16_t*>(a1 & ~(uintptr_t)1);
        r.sh1 = (uint32_t)(a1 & 1) * 8;
    } else {
        r.p1 = 0; r.sh1 = 0;
    }
}

// decode fetched words to the values attention reads (KVarN scale applied to low-bit rows)
__device__ __forceinline__ void decode_raw8(const SideView& v, const Raw8& r, int c0, float (&x)[8]) {
    const RowFmt f = r.sel ? v.ftail : v.fmain;
    if (f.kind != 0) {
        const uint32_t w0 = (uint32_t)r.w, w1 = (uint32_t)(r.w >> 32), w2 = (uint32_t)r.w2, w3 = (uint32_t)(r.w2 >> 32);
        if (f.kind == 1) {
            x[0] = __uint_as_float(w0 << 16); x[1] = __uint_as_float(w0 & 0xFFFF0000u);
            x[2] = __uint_as_float(w1 << 16); x[3] = __uint_as_float(w1 & 0xFFFF0000u);
            x[4] = __uint_as_float(w2 << 16); x[5] = __uint_as_float(w2 & 0xFFFF0000u);
            x[6] = __uint_as_float(w3 << 16); x[7] = __uint_as_float(w3 & 0xFFFF0000u);
        } else {
            x[0] = mma::h2f_lo(w0); x[1] = mma::h2f_hi(w0); x[2] = mma::h2f_lo(w1); x[3] = mma::h2f_hi(w1);
            x[4] = mma::h2f_lo(w2); x[5] = mma::h2f_hi(w2); x[6] = mma::h2f_lo(w3); x[7] = mma::h2f_hi(w3);
        }
        return;
    }
    const float d = mma::h2f_lo(r.dm);
    const float m = mma::h2f_hi(r.dm);
    const uint64_t p0 = r.w >> r.sh0;
    const uint32_t p1 = r.p1 >> r.sh1;
    const uint32_t m0 = (1u << f.w0) - 1, m1 = (1u << f.w1) - 1;
    const int off = 1 << (f.bits - 1);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int u = (int)(((uint32_t)(p0 >> (j * f.w0)) & m0) | (((p1 >> (j * f.w1)) & m1) << f.w0));
        x[j] = f.asym ? __fadd_rn(__fmul_rn(d, (float)u), m) : __fmul_rn(d, (float)(u - off));
    }
    if (v.scales && !r.sel) {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = __fmul_rn(v.scales[c0 + j], x[j]);
    }
}

// ---------------------------------------------------------------------------
// Fast dequantization for symmetric formats (qX_0, q8_0 tail) and the f16 tail: codes
// become exact fp16 integers with the 1024-magic unpack of the decode kernel, and the
// block scale is applied in fp16 as hi = RN(d*c), lo = d*c - hi (exact: d*c has at most
// 17 significant bits). K chunks come out in the k order (c0, c4, c1, c5, c2, c6, c3, c7)
// of each 8-channel chunk (the query is stored in the same order).
// ---------------------------------------------------------------------------
__host__ __device__ constexpr bool fast_fmt(int f) {
    return f == F_Q2_0 || f == F_Q3_0 || f == F_Q4_0 || f == F_Q5_0 || f == F_Q6_0 || f == F_Q8_0 || f == F_F16;
}

__device__ __forceinline__ void scale_pairs(const uint32_t (&p)[4], uint32_t dpair, uint32_t (&hi)[4],
                                            uint32_t (&lo)[4]) {
    const __half2 d2 = *reinterpret_cast<const __half2*>(&dpair);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 x = *reinterpret_cast<const __half2*>(&p[j]);
        const __half2 h = __hmul2_rn(x, d2);
        const __half2 l = __hfma2(x, d2, __hneg2(h));
        hi[j] = *reinterpret_cast<const uint32_t*>(&h);
        lo[j] = *reinterpret_cast<const uint32_t*>(&l);
    }
}

// K: channels 32b + 8t .. +7 of one row -> hi/lo in k order (0,4,1,5,2,6,3,7)
template <int F, int NB>
__device__ __forceinline__ void k_chunk_fast(const uint8_t* row, int b, int t, uint32_t (&out)[8]) {
    using namespace mma;
    if constexpr (F == F_F16) {
        const uint4 w = *reinterpret_cast<const uint4*>(row + 64 * b + 16 * t);
        out[0] = prmt(w.x, w.z, 0x5410u); out[1] = prmt(w.x, w.z, 0x7632u);
        out[2] = prmt(w.y, w.w, 0x5410u); out[3] = prmt(w.y, w.w, 0x7632u);
        out[4] = out[5] = out[6] = out[7] = 0u;
    } else {
        uint32_t p[4], hi[4], lo[4];
        k_pairs<F>(row, NB, b, t, p);
        const uint32_t d = reinterpret_cast<const uint16_t*>(row)[b];
        scale_pairs(p, d | (d << 16), hi, lo);
#pragma unroll
        for (int j = 0; j < 4; ++j) { out[j] = hi[j]; out[4 + j] = lo[j]; }
    }
}

// V: channels 32b + 4g .. +3 at 8 positions (rows r[0..7]) -> per channel 8 positions
// of hi (out[i][0..3]) and lo (out[i][4..7])
template <int F, int NB>
__device__ __forceinline__ void v_chunk_fast(const uint8_t* const (&r)[8], int b, int g, uint32_t (&out)[4][8]) {
    using namespace mma;
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
        uint32_t p[4];
        v_pairs<F>(r[2 * pp], r[2 * pp + 1], NB, b, g, p);
        if constexpr (F == F_F16) {
#pragma unroll
            for (int i = 0; i < 4; ++i) { out[i][pp] = p[i]; out[i][4 + pp] = 0u; }
        } else {
            const uint32_t da = reinterpret_cast<const uint16_t*>(r[2 * pp])[b];
            const uint32_t db = reinterpret_cast<const uint16_t*>(r[2 * pp + 1])[b];
            uint32_t hi[4], lo[4];
            scale_pairs(p, da | (db << 16), hi, lo);
#pragma unroll
            for (int i = 0; i < 4; ++i) { out[i][pp] = hi[i]; out[i][4 + pp] = lo[i]; }
        }
    }
}

// k order inside a K chunk: position p holds channel KPERM[p] of the chunk
__device__ __forceinline__ void kperm8(const float (&x)[8], float (&y)[8]) {
    y[0] = x[0]; y[1] = x[4]; y[2] = x[1]; y[3] = x[5]; y[4] = x[2]; y[5] = x[6]; y[6] = x[3]; y[7] = x[7];
}

// Position order inside a tile: K~ row r, S / P column r and V~^T k-slot r all hold
// position t0 + slot_pos(r), the (PN/8) x 8 transpose of the natural order. A thread that
// fills k-slots 8m .. 8m+7 of V~^T then reads staged rows m, m + PN/8, .., so lanes with
// consecutive m read consecutive rows (row strides are 16-byte multiples, so rows PN/8
// apart can share a shared-memory bank).
__host__ __device__ constexpr int slot_pos(int r) { return ((r & 7) * (PN / 8)) | (r >> 3); }
static_assert(PN % 8 == 0 && PN / 8 <= 8, "slot_pos needs 8-position groups");

constexpr int OWNER_WARPS = 4;                       // softmax / epilogue: one query row per thread
constexpr int DQ_WARPS = 11;                         // dequantization
constexpr int ISSUER_WARP = OWNER_WARPS + DQ_WARPS;  // lane 0 issues the MMAs and the bulk copies
static_assert(PTHREADS == 32 * (ISSUER_WARP + 1), "warp roles");

// bounded wait whose outcome is the same for every lane of the warp
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mma::mbar_wait(bar, parity, 2000000000ull, false)) != 0;
}
// the issuer's waits (single thread), polling: they sit on the tensor pipe's critical path
__device__ __forceinline__ bool poll_wait(uint64_t* bar, uint32_t parity) {
    return mma::mbar_wait(bar, parity, 2000000000ull, false);
}

template <int NB>
__global__ void __launch_bounds__(PTHREADS, 1) prefill_tc5(PrefillArgs a) {
    constexpr int D = 32 * NB;
    constexpr int CHUNKS = D / 8;                    // 8-channel chunks per row
    const size_t SH = (size_t)a.stage_half;
    const int KB = a.kbufs;
    const LayerView& lv = a.lv;
    extern __shared__ uint8_t raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* q_hi = sm;                              // Q hi [PM x D]; Q lo lives in TMEM
    uint8_t* k_base = q_hi + PM * D * 2;             // K~ [PN x D] hi, lo per buffer, 128-byte swizzle
    uint8_t* v_hi = k_base + (size_t)KB * 2 * PN * D * 2;   // V~^T [D x PN], 64-byte swizzle
    uint8_t* v_lo = v_hi + D * PN * 2;
    uint8_t* p_hi = v_lo + D * PN * 2;               // P [PM x PN], 64-byte swizzle
    uint8_t* p_lo = p_hi + PM * PN * 2;
    uint8_t* stage = p_lo + PM * PN * 2;             // 2 buffers x (K rows, V rows)
    uint64_t* bars = reinterpret_cast<uint64_t*>(stage + 4 * SH);
    uint64_t* st_full = bars;                        // [2] raw rows of a tile staged
    uint64_t* s_full = bars + 2;                     // [2] S of a tile in TMEM buffer t % 2
    uint64_t* s_empty = bars + 4;                    // [2] owners have read that S buffer
    uint64_t* k_full = bars + 6;                     // [2] K~ buffer written
    uint64_t* k_empty = bars + 8;                    // [2] S MMAs done reading that K~ buffer
    uint64_t* v_full = bars + 10;                    // V~^T written (and the staging buffer consumed)
    uint64_t* p_full = bars + 11;                    // P written
    uint64_t* o_done = bars + 12;                    // P V~ MMAs done
    volatile int* fault_flag = reinterpret_cast<volatile int*>(bars + 13);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool owner = warp < OWNER_WARPS;           // owns TMEM lane / query row tid
    const int G = lv.G, H = lv.H;
    const int h = blockIdx.y, b = blockIdx.z / a.splits, sp = blockIdx.z % a.splits;
    const int rows_total = a.C * G;
    const int row0 = blockIdx.x * PM;
    const int r = row0 + (tid & (PM - 1));           // query row of an owner thread
    const bool row_ok = owner && r < rows_total;
    const int ci = row_ok ? r / G : 0;               // chunk row
    const int gi = row_ok ? r % G : 0;
    const int n = (int)a.n;                          // positions < 2^31 (checked on the host)
    const int pos0 = n - a.C;
    const int my_limit = row_ok ? pos0 + ci : -1;    // last visible position
    const int last_row = min(rows_total - 1, row0 + PM - 1);
    const int tile_limit = pos0 + last_row / G;      // last position any row sees
    const int first_row_limit = pos0 + row0 / G;
    const SideView kside = side_view(lv, b, h, 0);
    const SideView vside = side_view(lv, b, h, 1);
    const int W = lv.W;
    const int ring0 = W > 0 ? n - W : n;             // first position held in the ring
    // this CTA's key tiles: [t_lo, t_lo + n_tiles) of the M-tile's tiles_all (positions from
    // tb = t_lo * PN; the host splits only when every split keeps 32 tiles or more); tile
    // indices below count from t_lo
    const int tiles_all = tile_limit / PN + 1;
    const int t_lo = (int)((long long)tiles_all * sp / a.splits);
    const int n_tiles = (int)((long long)tiles_all * (sp + 1) / a.splits) - t_lo;
    const int tb = t_lo * PN;
    const long long rows_all = (long long)lv.B * a.C * G * H;
    const long long orow_idx = ((long long)b * a.C + ci) * (G * H) + (long long)h * G + gi;
    // where the row's O goes: the output row, or this split's partial
    float* const orow = a.splits > 1 ? a.part + ((long long)sp * rows_all + orow_idx) * D : a.out + orow_idx * D;
    // K~ and V~ enter the MMAs scaled by 2^-ek, 2^-ev (exponents from the bounds the appends
    // keep, 0 for ordinary ranges) so that their fp16 hi + lo parts neither overflow nor lose
    // their low part to fp16's subnormal range; S and O are scaled back exactly
    const int ek = fp16_exponent(__uint_as_float(lv.stats[((long long)(b * H + h) * 2 + 0) * 2 + 1]), -120, 120);
    const int ev = fp16_exponent(__uint_as_float(lv.stats[((long long)(b * H + h) * 2 + 1) * 2 + 1]), -120, 120);
    const float kmul = __uint_as_float((uint32_t)(127 - ek) << 23);
    const float vmul = __uint_as_float((uint32_t)(127 - ev) << 23);

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mma::mbar_init(&st_full[i], 1);
            mma::mbar_init(&s_full[i], 1);
            mma::mbar_init(&s_empty[i], OWNER_WARPS);
            mma::mbar_init(&k_full[i], DQ_WARPS);
            mma::mbar_init(&k_empty[i], 1);
        }
        mma::mbar_init(v_full, DQ_WARPS);
        mma::mbar_init(p_full, OWNER_WARPS);
        mma::mbar_init(o_done, 1);
        *fault_flag = 0;
        mma::fence_mbar_init();
    }
    if (warp == 0) { t5::tmem_alloc(tmem_slot, 512); t5::tmem_relinquish(); }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // S of buffer sb: two partial sums over the channel halves (columns 2 PN sb + [0, PN) and
    // 2 PN sb + [PN, 2 PN)), added with IEEE fp32 adds by the owners: the tensor-memory
    // accumulation then runs over half the k-steps, which halves its rounding error at
    // large logits
    const uint32_t t_s = tmem;                       // S: columns [0, 4 PN)
    const uint32_t t_qlo = tmem + 4 * PN;            // Q lo: columns [4 PN, 4 PN + D/2)
    const uint32_t t_o = tmem + 256;                 // O: columns [256, 256 + D)
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;

    // bulk copies of tile `tile`'s raw rows into staging buffer tile % 2 (issuer lane)
    int st_last[2] = {-1, -1};                       // last tile staged per buffer
    auto issue_stage = [&](int tile) {
        const int t0 = tb + tile * PN;
        const int tl = min(t0 + PN - 1, tile_limit);
        const int nm = max(0, min(tl + 1, ring0) - t0);       // rows from the low-bit store
        const int nr = (tl + 1 - t0) - nm;                    // rows from the ring
        uint64_t* bar = &st_full[tile & 1];
        uint32_t bytes = 0;
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
            const RowFmt fm = kv ? vside.fmain : kside.fmain;
            const RowFmt ft = kv ? vside.ftail : kside.ftail;
            if (nm > 0) bytes += (uint32_t)nm * fm.stride;
            if (nr > 0) bytes += (uint32_t)nr * ft.stride;
        }
        mma::mbar_arrive_expect_tx(bar, bytes);
        if (tile & 1) st_last[1] = tile; else st_last[0] = tile;
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
            const SideView v = kv ? vside : kside;
            uint8_t* dst = stage + (size_t)(tile & 1) * 2 * SH + kv * SH;
            if (nm > 0) {
                const uint32_t cb = (uint32_t)nm * v.fmain.stride;
                mma::bulk_g2s(dst, v.main + (long long)t0 * v.fmain.stride, cb, bar);
                dst += cb;
            }
            if (nr > 0) {
                const int p = t0 + nm;                         // first ring position
                const int s0 = p % W;
                const int c1 = min(nr, W - s0);
                mma::bulk_g2s(dst, v.ring + (long long)s0 * v.ftail.stride, (uint32_t)c1 * v.ftail.stride, bar);
                if (nr > c1)
                    mma::bulk_g2s(dst + (size_t)c1 * v.ftail.stride, v.ring, (uint32_t)(nr - c1) * v.ftail.stride, bar);
            }
        }
    };
    const bool issuer = warp == ISSUER_WARP && lane == 0;
    if (issuer) {
        issue_stage(0);
        if (n_tiles > 1) issue_stage(1);
    }

    // ---- query rows: Q hi -> shared memory, Q lo -> TMEM (owners write their own row). A row
    // is normalised by a power of two 2^-eq (eq = 0 for ordinary ranges); its scores are
    // multiplied back by 2^(eq + ek).
    float s_mul = 1.f;
    if (owner) {
        const float* qr = a.q + (((long long)b * a.C + ci) * (G * H) + (long long)h * G + gi) * D;
        float qn = 1.f;
        if (row_ok) {
            float mq = 0.f;
            for (int c = 0; c < D; c += 4) {
                const float4 p = *reinterpret_cast<const float4*>(qr + c);
                mq = fmaxf(mq, fmaxf(fmaxf(fabsf(p.x), fabsf(p.y)), fmaxf(fabsf(p.z), fabsf(p.w))));
            }
            const int eq = fp16_exponent(mq * fabsf(a.qscale), -120, 120);
            qn = __uint_as_float((uint32_t)(127 - eq) << 23);
            s_mul = __uint_as_float((uint32_t)(127 + eq) << 23) * __uint_as_float((uint32_t)(127 + ek) << 23);
        }
#pragma unroll 1
        for (int c64 = 0; c64 < D; c64 += 64) {      // 64 k-values = 32 TMEM columns
            float cols[32];
#pragma unroll
            for (int k0 = 0; k0 < 64; k0 += 8) {
                float x[8], y[8];
                if (row_ok) {
                    const float4 p = *reinterpret_cast<const float4*>(qr + c64 + k0);
                    const float4 v = *reinterpret_cast<const float4*>(qr + c64 + k0 + 4);
                    x[0] = p.x; x[1] = p.y; x[2] = p.z; x[3] = p.w; x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[j] = (x[j] * a.qscale) * qn;
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[j] = 0.f;
                }
                kperm8(x, y);
                __align__(16) __half hh[8], ll[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) split16(y[j], hh[j], ll[j]);
                *reinterpret_cast<uint4*>(q_hi + t5::sw128_offset(tid, c64 + k0, PM)) = *reinterpret_cast<const uint4*>(hh);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    cols[k0 / 2 + j] = __uint_as_float((uint32_t)__half_as_ushort(ll[2 * j]) |
                                                       ((uint32_t)__half_as_ushort(ll[2 * j + 1]) << 16));
            }
            t5::tmem_st32(t_qlo + lane_off + c64 / 2, cols);
        }
        t5::fence_proxy_async();
    }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();

    // Tile modes (uniform over the CTA): 1 = every position in the low-bit store and its
    // format has a fast path, 2 = every position in the ring with a fast tail format,
    // 0 = generic decode (mixed tiles, asymmetric / bf16 formats, KVarN).
    auto tile_mode = [&](int t0, const SideView& v, int e) -> int {
        if (e != 0) return 0;                        // scaled values take the generic path
        const int last = min(t0 + PN - 1, tile_limit);
        if (last < ring0 && !v.scales && fast_fmt(v.fmain.id)) return 1;
        if (t0 >= ring0 && fast_fmt(v.ftail.id)) return 2;
        return 0;
    };
    // staged row of position t (clamped to the tile's last position)
    auto srow = [&](int kv, int t0, int t, uint32_t& sel) -> const uint8_t* {
        const RowFmt fm = kv ? vside.fmain : kside.fmain;
        const RowFmt ft = kv ? vside.ftail : kside.ftail;
        const int tl = min(t0 + PN - 1, tile_limit);
        t = min(t, tl);
        const int nm = max(0, min(tl + 1, ring0) - t0);
        const uint8_t* base = stage + (size_t)(((t0 - tb) / PN) & 1) * 2 * SH + kv * SH;
        if (t - t0 < nm) { sel = 0; return base + (size_t)(t - t0) * fm.stride; }
        sel = 1;
        return base + (size_t)nm * fm.stride + (size_t)(t - t0 - nm) * ft.stride;
    };
    auto set_fault = [&]() { *fault_flag = 1; };

    float m_run = -INFINITY, l_run = 0.f;
    float gcorr = 1.f;                               // owners: pending rescale of the folded partial
    int s_last = -1, o_last = -1;                    // issuer: last tile whose S / P V~ MMAs were committed

    if (owner) {
        // ======================= softmax: S(t) -> P(t), running max and sum of the row
        for (int t = 0; t < n_tiles; ++t) {
            if (*fault_flag) break;
            const int t0 = tb + t * PN;
            const int sb = t & 1;
            if (!warp_wait(&s_full[sb], (t >> 1) & 1)) { set_fault(); break; }
            t5::fence_after_sync();
            float sv[32], sv2[32];
            t5::tmem_ld32(t_s + 2 * PN * sb + lane_off, sv);
            t5::tmem_ld32(t_s + 2 * PN * sb + PN + lane_off, sv2);
            t5::fence_before_sync();
            __syncwarp();
            if (lane == 0) mma::mbar_arrive(&s_empty[sb]);
#pragma unroll
            for (int i = 0; i < PN; ++i) sv[i] += sv2[i];
            if (s_mul != 1.f) {
#pragma unroll
                for (int i = 0; i < PN; ++i) sv[i] *= s_mul;
            }
            const bool full = t0 + PN - 1 <= first_row_limit;
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < PN; ++i) {
                if (!full && t0 + slot_pos(i) > my_limit) sv[i] = -INFINITY;
                mx = fmaxf(mx, sv[i]);
            }
            const bool raise = mx > m_run + PF_RESCALE || (m_run == -INFINITY && mx > -INFINITY);
            const float corr = !raise ? 1.f : ((m_run == -INFINITY) ? 0.f : mma::ex2(m_run - mx));
            if (raise) {
                l_run *= corr;
                m_run = mx;
            }
            // P and O are read by the previous tile's P V~ MMAs: wait for them
            if (t > 0) {
                if (!warp_wait(o_done, (t - 1) & 1)) { set_fault(); break; }
                t5::fence_after_sync();
            }
            if (t > 0 && t % PF_FOLD == 0) {
                // fold: O in TMEM holds tiles [t - PF_FOLD, t); add it to the partial in the
                // output row, apply this tile's correction; P V~(t) then starts afresh
                const bool first = t == PF_FOLD;
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    float o[32];
                    t5::tmem_ld32(t_o + lane_off + c, o);      // warp-collective
                    if (row_ok) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            float4 g4 = first ? make_float4(0.f, 0.f, 0.f, 0.f)
                                              : *reinterpret_cast<const float4*>(orow + c + i);
                            g4.x = (g4.x * gcorr + o[i]) * corr;
                            g4.y = (g4.y * gcorr + o[i + 1]) * corr;
                            g4.z = (g4.z * gcorr + o[i + 2]) * corr;
                            g4.w = (g4.w * gcorr + o[i + 3]) * corr;
                            *reinterpret_cast<float4*>(orow + c + i) = g4;
                        }
                    }
                }
                gcorr = 1.f;
            } else {
                gcorr *= corr;                           // the folded partial follows the max lazily
                // TMEM loads/stores are warp-collective: rescale O when any lane of the warp
                // raised its max (lanes that did not use factor 1)
                if (t > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        float o[32];
                        t5::tmem_ld32(t_o + lane_off + c, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= corr;
                        t5::tmem_st32(t_o + lane_off + c, o);
                    }
                }
            }
            float ps = 0.f;
#pragma unroll
            for (int i = 0; i < PN; ++i) {
                const float p = (m_run == -INFINITY || sv[i] == -INFINITY) ? 0.f : mma::ex2(sv[i] - m_run);
                sv[i] = p;
                ps += p;
            }
#pragma unroll
            for (int k0 = 0; k0 < PN; k0 += 8) {
                float x8[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) x8[j] = sv[k0 + j];
                store_chunk64(p_hi, p_lo, tid, k0, x8);
            }
            l_run += ps;
            t5::fence_proxy_async();
            t5::fence_before_sync();
            __syncwarp();
            if (lane == 0) mma::mbar_arrive(p_full);
        }
    } else if (warp < ISSUER_WARP) {
        // ======================= dequantization: staged rows -> K~(t), V~^T(t)
        const int dt = tid - 32 * OWNER_WARPS;
        constexpr int KUNITS = PN * CHUNKS;              // (row, 8-channel chunk)
        constexpr int VUNITS = (PN / 8) * 8 * NB;        // (8 positions, 4 channels)
        constexpr int GUNITS = (PN / 8) * CHUNKS * 2;    // generic V: (8 positions, 4 channels)
        for (int t = 0; t < n_tiles; ++t) {
            if (*fault_flag) break;
            const int t0 = tb + t * PN;
            // K~ buffer of this tile: free once the S MMAs of tile t - KB have read it
            const int kb = KB == 2 ? (t & 1) : 0;
            uint8_t* k_hi = k_base + (size_t)kb * 2 * PN * D * 2;
            uint8_t* k_lo = k_hi + PN * D * 2;
            bool ok = warp_wait(&st_full[t & 1], (t >> 1) & 1);
            if (ok && t >= KB) ok = warp_wait(&k_empty[kb], (KB == 2 ? (t >> 1) - 1 : t - 1) & 1);
            if (!ok) { set_fault(); break; }
            {
                const int kmode = tile_mode(t0, kside, ek);
                const int fid = kmode == 1 ? kside.fmain.id : kside.ftail.id;
                for (int u = dt; u < KUNITS; u += 32 * DQ_WARPS) {
                    const int kr = u / CHUNKS, ch = u % CHUNKS;
                    uint32_t sel;
                    const uint8_t* row = srow(0, t0, t0 + slot_pos(kr), sel);
                    if (kmode != 0) {
                        uint32_t out[8];
                        const int cb = ch >> 2, ct = ch & 3;
                        switch (fid) {
                            case F_Q2_0: k_chunk_fast<F_Q2_0, NB>(row, cb, ct, out); break;
                            case F_Q3_0: k_chunk_fast<F_Q3_0, NB>(row, cb, ct, out); break;
                            case F_Q4_0: k_chunk_fast<F_Q4_0, NB>(row, cb, ct, out); break;
                            case F_Q5_0: k_chunk_fast<F_Q5_0, NB>(row, cb, ct, out); break;
                            case F_Q6_0: k_chunk_fast<F_Q6_0, NB>(row, cb, ct, out); break;
                            case F_Q8_0: k_chunk_fast<F_Q8_0, NB>(row, cb, ct, out); break;
                            default: k_chunk_fast<F_F16, NB>(row, cb, ct, out); break;
                        }
                        const uint32_t off = t5::sw128_offset(kr, 8 * ch, PN);
                        *reinterpret_cast<uint4*>(k_hi + off) = make_uint4(out[0], out[1], out[2], out[3]);
                        *reinterpret_cast<uint4*>(k_lo + off) = make_uint4(out[4], out[5], out[6], out[7]);
                    } else {
                        Raw8 rk;
                        fetch8_row(row, sel ? kside.ftail : kside.fmain, sel, 8 * ch, NB, rk);
                        float x[8], y[8];
                        decode_raw8(kside, rk, 8 * ch, x);
#pragma unroll
                        for (int j = 0; j < 8; ++j) x[j] *= kmul;
                        kperm8(x, y);
                        store_chunk(k_hi, k_lo, kr, 8 * ch, PN, y);
                    }
                }
            }
            t5::fence_proxy_async();
            __syncwarp();
            if (lane == 0) mma::mbar_arrive(&k_full[kb]);
            if (t > 0 && !warp_wait(o_done, (t - 1) & 1)) { set_fault(); break; }   // P V~(t-1) done reading V~^T
            const int vmode = tile_mode(t0, vside, ev);
            if (vmode != 0) {
                const int vfid = vmode == 1 ? vside.fmain.id : vside.ftail.id;
                for (int u = dt; u < VUNITS; u += 32 * DQ_WARPS) {
                    const int pg = u % (PN / 8), g = (u / (PN / 8)) & 7, vb = u / (PN / 8) / 8;
                    const uint8_t* rr[8];
                    uint32_t sel;
#pragma unroll
                    for (int j = 0; j < 8; ++j) rr[j] = srow(1, t0, t0 + pg + (PN / 8) * j, sel);
                    uint32_t o[4][8];
                    switch (vfid) {
                        case F_Q2_0: v_chunk_fast<F_Q2_0, NB>(rr, vb, g, o); break;
                        case F_Q3_0: v_chunk_fast<F_Q3_0, NB>(rr, vb, g, o); break;
                        case F_Q4_0: v_chunk_fast<F_Q4_0, NB>(rr, vb, g, o); break;
                        case F_Q5_0: v_chunk_fast<F_Q5_0, NB>(rr, vb, g, o); break;
                        case F_Q6_0: v_chunk_fast<F_Q6_0, NB>(rr, vb, g, o); break;
                        case F_Q8_0: v_chunk_fast<F_Q8_0, NB>(rr, vb, g, o); break;
                        default: v_chunk_fast<F_F16, NB>(rr, vb, g, o); break;
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t off = t5::sw64_offset(32 * vb + 4 * g + c, 8 * pg);
                        *reinterpret_cast<uint4*>(v_hi + off) = make_uint4(o[c][0], o[c][1], o[c][2], o[c][3]);
                        *reinterpret_cast<uint4*>(v_lo + off) = make_uint4(o[c][4], o[c][5], o[c][6], o[c][7]);
                    }
                }
            } else {
                // generic: decode 8 positions x 8 channels, keep one half (4 channels)
                for (int u = dt; u < GUNITS; u += 32 * DQ_WARPS) {
                    const int tg = u % (PN / 8), cc = (u / (PN / 8)) % CHUNKS, e4 = u / (PN / 8) / CHUNKS;
                    float xv[8][4];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int tp = t0 + tg + (PN / 8) * j;
                        uint32_t sel;
                        const uint8_t* row = srow(1, t0, tp, sel);
                        Raw8 rv;
                        fetch8_row(row, sel ? vside.ftail : vside.fmain, sel, 8 * cc, NB, rv);
                        float x[8];
                        decode_raw8(vside, rv, 8 * cc, x);
                        const bool live = tp <= tile_limit;
#pragma unroll
                        for (int e = 0; e < 4; ++e) xv[j][e] = live ? x[4 * e4 + e] * vmul : 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float y[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) y[j] = xv[j][e];
                        store_chunk64(v_hi, v_lo, 8 * cc + 4 * e4 + e, 8 * tg, y);
                    }
                }
            }
            t5::fence_proxy_async();
            __syncwarp();
            if (lane == 0) mma::mbar_arrive(v_full);          // also: this tile's staging is consumed
        }
    } else if (issuer) {
        // ======================= MMA issue and staging
        const uint32_t idesc_s = t5::idesc_f16(PM, PN);
        const uint32_t idesc_o = t5::idesc_f16(PM, D);
        // descriptors advance by (bytes >> 4) in their start-address field
        const uint64_t dq0 = t5::desc_sw128(t5::smem_addr(q_hi));
        const uint64_t dkb0 = t5::desc_sw128(t5::smem_addr(k_base));     // K~ buffer 0, hi part
        const uint64_t dkstep = (uint64_t)((PN * D * 2) >> 4);             // hi -> lo, and per buffer 2 steps
        const uint64_t dph0 = t5::desc_sw64(t5::smem_addr(p_hi)), dpl0 = t5::desc_sw64(t5::smem_addr(p_lo));
        const uint64_t dvh0 = t5::desc_sw64(t5::smem_addr(v_hi)), dvl0 = t5::desc_sw64(t5::smem_addr(v_lo));
        // S MMAs of tile t (waits for K~(t) and for the owners to have read S(t - 2))
        auto issue_s = [&](int t) -> bool {
            const int sb = t & 1;
            const int kb = KB == 2 ? (t & 1) : 0;
            const uint64_t dkh0 = dkb0 + (uint64_t)(2 * kb) * dkstep, dkl0 = dkh0 + dkstep;
            bool ok = poll_wait(&k_full[kb], (KB == 2 ? (t >> 1) : t) & 1);
            if (ok && t >= 2) ok = poll_wait(&s_empty[sb], ((t >> 1) - 1) & 1);
            if (!ok) return false;
            t5::fence_after_sync();
            const uint32_t ts = t_s + 2 * PN * sb;
            constexpr int KH = D / 32;                 // k-steps per channel half
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t dk = (uint64_t)(((k >> 2) * PM * 128 + (k & 3) * 32) >> 4);
                const uint64_t dkk = (uint64_t)(((k >> 2) * PN * 128 + (k & 3) * 32) >> 4);
                t5::mma_f16_ss(ts + (k >= KH ? PN : 0), dq0 + dk, dkh0 + dkk, idesc_s, (k % KH) > 0);
            }
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t dk = (uint64_t)(((k >> 2) * PM * 128 + (k & 3) * 32) >> 4);
                const uint64_t dkk = (uint64_t)(((k >> 2) * PN * 128 + (k & 3) * 32) >> 4);
                t5::mma_f16_ss(ts + (k >= KH ? PN : 0), dq0 + dk, dkl0 + dkk, idesc_s, true);
            }
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t dkk = (uint64_t)(((k >> 2) * PN * 128 + (k & 3) * 32) >> 4);
                t5::mma_f16_ts(ts + (k >= KH ? PN : 0), t_qlo + 8 * k, dkh0 + dkk, idesc_s, true);
            }
            t5::mma_commit(&s_full[sb]);
            t5::mma_commit(&k_empty[kb]);
            s_last = t;
            return true;
        };
        // P V~ MMAs of tile t (waits for V~^T(t) and P(t)), then refill its staging buffer
        auto issue_pv = [&](int t) -> bool {
            bool ok = poll_wait(v_full, t & 1);
            if (ok) ok = poll_wait(p_full, t & 1);
            if (!ok) return false;
            t5::fence_after_sync();
#pragma unroll
            for (int k = 0; k < PN / 16; ++k) {
                const uint64_t dk = (uint64_t)((k * 32) >> 4);
                t5::mma_f16_ss(t_o, dph0 + dk, dvh0 + dk, idesc_o, t % PF_FOLD != 0 || k > 0);
            }
#pragma unroll
            for (int k = 0; k < PN / 16; ++k) {
                const uint64_t dk = (uint64_t)((k * 32) >> 4);
                t5::mma_f16_ss(t_o, dph0 + dk, dvl0 + dk, idesc_o, true);
            }
#pragma unroll
            for (int k = 0; k < PN / 16; ++k) {
                const uint64_t dk = (uint64_t)((k * 32) >> 4);
                t5::mma_f16_ss(t_o, dpl0 + dk, dvh0 + dk, idesc_o, true);
            }
            t5::mma_commit(o_done);
            o_last = t;
            if (t + 2 < n_tiles) issue_stage(t + 2);   // this tile's staging buffer is consumed
            return true;
        };
        // S(t) then P V~(t): P V~(t) is queued ahead of S(t + 1) on the tensor pipe, so the
        // V~^T buffer it reads is released as early as possible
        bool ok = true;
        for (int t = 0; ok && t < n_tiles; ++t) {
            if (*fault_flag) break;
            ok = issue_s(t);
            if (ok) ok = issue_pv(t);
        }
        if (!ok) set_fault();
    }

    // ---- epilogue: O / l -> out (TMEM loads by whole owner warps; only real rows store)
    __syncthreads();
    if (owner && !*fault_flag) {
        if (!warp_wait(o_done, (n_tiles - 1) & 1)) set_fault();
        t5::fence_after_sync();
    }
    __syncthreads();
    const bool any_fault = *fault_flag != 0;
    if (owner && !any_fault) {
        const float vsc = __uint_as_float((uint32_t)(127 + ev) << 23);
        // one split: O / l; several: O unnormalised, with the row's max and sum beside it
        const float inv = !row_ok ? 0.f : (a.splits > 1 ? vsc : vsc / l_run);
        if (a.splits > 1 && row_ok) {
            float* ml = a.part + (long long)a.splits * rows_all * D + ((long long)sp * rows_all + orow_idx) * 2;
            ml[0] = m_run;
            ml[1] = l_run;
        }
        const bool folded = n_tiles > PF_FOLD;      // a partial of earlier tiles is in orow
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
            float o[32];
            t5::tmem_ld32(t_o + lane_off + c, o);
            if (row_ok) {
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 g4 = folded ? *reinterpret_cast<const float4*>(orow + c + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                    g4.x = (g4.x * gcorr + o[i]) * inv;
                    g4.y = (g4.y * gcorr + o[i + 1]) * inv;
                    g4.z = (g4.z * gcorr + o[i + 2]) * inv;
                    g4.w = (g4.w * gcorr + o[i + 3]) * inv;
                    *reinterpret_cast<float4*>(orow + c + i) = g4;
                }
            }
        }
    } else if (row_ok && any_fault) {
        if (tid == 0) atomicOr(lv.status, STATUS_WAIT_TIMEOUT);
        for (int c = 0; c < D; ++c) orow[c] = __int_as_float(0x7fc00000);
    }
    if (any_fault && issuer) {
        // copies and MMAs may still be in flight: give each a bounded wait before the
        // shared and tensor memory are released
        for (int i = 0; i < 2; ++i)
            if (st_last[i] >= 0) mma::mbar_wait(&st_full[i], (st_last[i] >> 1) & 1, 50000000ull);
        if (s_last >= 0) mma::mbar_wait(&s_full[s_last & 1], (s_last >> 1) & 1, 50000000ull);
        if (o_last >= 0) mma::mbar_wait(o_done, o_last & 1, 50000000ull);
    }
    t5::fence_before_sync();
    __syncthreads();
    if (warp == 0) t5::tmem_dealloc(tmem, 512);
}

// ===========================================================================
// Staged prefill: each K~ / V~^T tile is dequantized once per (batch, kv head) into a
// workspace image laid out exactly as the shared-memory operand tiles, then every M-tile CTA
// of that head streams the images with bulk copies instead of dequantizing them itself (the
// 128-row M-tiles of one head all read the same tiles: dequantizing in each of them made the
// prefill bound by its dequantization warps).
//
// Image of tile t (positions t*PN .. t*PN + PN - 1 in the transposed in-tile order
// slot_pos, positions past the end clamped to the last cached one): K~ as one 2PN x D fp16
// operand, 128-byte-swizzled K-major, whose rows 0 .. PN-1 are the hi parts and rows
// PN .. 2PN-1 the lo parts of the tile's positions (so one N = 2PN MMA multiplies a Q
// fragment by both); then V~^T hi | V~^T lo (each D x PN fp16, 64-byte swizzle); scaled by the
// same powers of two 2^-ek, 2^-ev as the on-the-fly kernel.
// ===========================================================================
__host__ __device__ constexpr size_t tile_image_bytes(int D) { return (size_t)4 * PN * D * 2; }

template <int NB>
__global__ void __launch_bounds__(256) prefill_tiles(LayerView lv, long long n, uint8_t* img, long long img_tiles) {
    constexpr int D = 32 * NB;
    constexpr int CHUNKS = D / 8;
    constexpr int KUNITS = PN * CHUNKS;
    constexpr int VUNITS = (PN / 8) * 8 * NB;
    constexpr int GUNITS = (PN / 8) * CHUNKS * 2;
    const int h = blockIdx.y, b = blockIdx.z;
    const long long t = blockIdx.x;
    const int t0 = (int)(t * PN);
    const int last = (int)n - 1;
    const SideView kside = side_view(lv, b, h, 0);
    const SideView vside = side_view(lv, b, h, 1);
    const int W = lv.W;
    const int ring0 = W > 0 ? (int)n - W : (int)n;
    const int ek = fp16_exponent(__uint_as_float(lv.stats[((long long)(b * lv.H + h) * 2 + 0) * 2 + 1]), -120, 120);
    const int ev = fp16_exponent(__uint_as_float(lv.stats[((long long)(b * lv.H + h) * 2 + 1) * 2 + 1]), -120, 120);
    const float kmul = __uint_as_float((uint32_t)(127 - ek) << 23);
    const float vmul = __uint_as_float((uint32_t)(127 - ev) << 23);
    uint8_t* base = img + ((long long)(b * lv.H + h) * img_tiles + t) * tile_image_bytes(D);
    uint8_t* k_hl = base;                            // [D/64][hi rows | lo rows][128 B]
    uint8_t* v_hi = base + 2 * PN * D * 2;
    uint8_t* v_lo = base + 3 * PN * D * 2;
    // row of position p (clamped to the last cached position): the low-bit store or the ring
    auto grow = [&](const SideView& v, int p, uint32_t& sel) -> const uint8_t* {
        p = min(p, last);
        if (p < ring0) { sel = 0; return v.main + (long long)p * v.fmain.stride; }
        sel = 1;
        return v.ring + (long long)(p % W) * v.ftail.stride;
    };
    auto mode = [&](const SideView& v, int e) -> int {
        if (e != 0) return 0;
        const int tl = min(t0 + PN - 1, last);
        if (tl < ring0 && !v.scales && fast_fmt(v.fmain.id)) return 1;
        if (t0 >= ring0 && fast_fmt(v.ftail.id)) return 2;
        return 0;
    };
    const int kmode = mode(kside, ek);
    const int kfid = kmode == 1 ? kside.fmain.id : kside.ftail.id;
    for (int u = threadIdx.x; u < KUNITS; u += blockDim.x) {
        const int kr = u / CHUNKS, ch = u % CHUNKS;
        uint32_t sel;
        const uint8_t* row = grow(kside, t0 + slot_pos(kr), sel);
        if (kmode != 0) {
            uint32_t out[8];
            const int cb = ch >> 2, ct = ch & 3;
            switch (kfid) {
                case F_Q2_0: k_chunk_fast<F_Q2_0, NB>(row, cb, ct, out); break;
                case F_Q3_0: k_chunk_fast<F_Q3_0, NB>(row, cb, ct, out); break;
                case F_Q4_0: k_chunk_fast<F_Q4_0, NB>(row, cb, ct, out); break;
                case F_Q5_0: k_chunk_fast<F_Q5_0, NB>(row, cb, ct, out); break;
                case F_Q6_0: k_chunk_fast<F_Q6_0, NB>(row, cb, ct, out); break;
                case F_Q8_0: k_chunk_fast<F_Q8_0, NB>(row, cb, ct, out); break;
                default: k_chunk_fast<F_F16, NB>(row, cb, ct, out); break;
            }
            const uint32_t off = t5::sw128_offset(kr, 8 * ch, 2 * PN);
            *reinterpret_cast<uint4*>(k_hl + off) = make_uint4(out[0], out[1], out[2], out[3]);
            *reinterpret_cast<uint4*>(k_hl + off + PN * 128) = make_uint4(out[4], out[5], out[6], out[7]);
        } else {
            Raw8 rk;
            fetch8_row(row, sel ? kside.ftail : kside.fmain, sel, 8 * ch, NB, rk);
            float x[8], y[8];
            decode_raw8(kside, rk, 8 * ch, x);
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] *= kmul;
            kperm8(x, y);
            store_chunk(k_hl, k_hl + PN * 128, kr, 8 * ch, 2 * PN, y);   // lo row PN + kr
        }
    }
    const int vmode = mode(vside, ev);
    if (vmode != 0) {
        const int vfid = vmode == 1 ? vside.fmain.id : vside.ftail.id;
        for (int u = threadIdx.x; u < VUNITS; u += blockDim.x) {
            const int pg = u % (PN / 8), g = (u / (PN / 8)) & 7, vb = u / (PN / 8) / 8;
            const uint8_t* rr[8];
            uint32_t sel;
#pragma unroll
            for (int j = 0; j < 8; ++j) rr[j] = grow(vside, t0 + pg + (PN / 8) * j, sel);
            uint32_t o[4][8];
            switch (vfid) {
                case F_Q2_0: v_chunk_fast<F_Q2_0, NB>(rr, vb, g, o); break;
                case F_Q3_0: v_chunk_fast<F_Q3_0, NB>(rr, vb, g, o); break;
                case F_Q4_0: v_chunk_fast<F_Q4_0, NB>(rr, vb, g, o); break;
                case F_Q5_0: v_chunk_fast<F_Q5_0, NB>(rr, vb, g, o); break;
                case F_Q6_0: v_chunk_fast<F_Q6_0, NB>(rr, vb, g, o); break;
                case F_Q8_0: v_chunk_fast<F_Q8_0, NB>(rr, vb, g, o); break;
                default: v_chunk_fast<F_F16, NB>(rr, vb, g, o); break;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t off = t5::sw64_offset(32 * vb + 4 * g + c, 8 * pg);
                *reinterpret_cast<uint4*>(v_hi + off) = make_uint4(o[c][0], o[c][1], o[c][2], o[c][3]);
                *reinterpret_cast<uint4*>(v_lo + off) = make_uint4(o[c][4], o[c][5], o[c][6], o[c][7]);
            }
        }
    } else {
        for (int u = threadIdx.x; u < GUNITS; u += blockDim.x) {
            const int tg = u % (PN / 8), cc = (u / (PN / 8)) % CHUNKS, e4 = u / (PN / 8) / CHUNKS;
            float xv[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int tp = t0 + tg + (PN / 8) * j;
                uint32_t sel;
                const uint8_t* row = grow(vside, tp, sel);
                Raw8 rv;
                fetch8_row(row, sel ? vside.ftail : vside.fmain, sel, 8 * cc, NB, rv);
                float x[8];
                decode_raw8(vside, rv, 8 * cc, x);
                const bool live = tp <= last;
#pragma unroll
                for (int e = 0; e < 4; ++e) xv[j][e] = live ? x[4 * e4 + e] * vmul : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float y[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) y[j] = xv[j][e];
                store_chunk64(v_hi, v_lo, 8 * cc + 4 * e4 + e, 8 * tg, y);
            }
        }
    }
}

struct StagedArgs {
    LayerView lv;
    const float* q;
    float* out;
    float qscale;
    long long n;
    int C;
    const uint8_t* img;           // tile images of every (b, h)
    long long img_tiles;          // tiles per (b, h) in the image area
    int splits;                   // key-range splits per M-tile (1: rows finished in place)
    float* part;                  // splits > 1: [splits][B * C * Hq][D] unnormalised O, then
                                  // [splits][B * C * Hq][2] (running max, row sum)
};

// Warp roles of the staged kernel: 8 softmax / epilogue warps own the 128 query rows in pairs
// (warps w and w + 4 share TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31, one row per lane: both
// compute the row's running max from all of S, each turns its half of the tile's columns
// into P and handles its half of the O columns), two warps whose lane 0 issue MMAs (one the S'
// and P V~ MMAs, the other the S'' MMAs: an MMA occupies its issuing thread for ~50 cycles
// whatever its size, so narrow MMAs from two threads overlap where one thread's would queue)
// and one whose lane 0 issues the bulk copies. MMA issue stalls while the tensor pipe's short
// queue is full, so the issuing threads do nothing else that could let the queue run dry.
constexpr int SP_OWNERS = 8;
constexpr int SP_THREADS = 32 * (SP_OWNERS + 3);
constexpr int SP_KBUF = 3;                                 // K~ buffers: fetched two tiles ahead
__host__ __device__ constexpr size_t sp_smem(int D) {
    return 1024 /* alignment slack */ + (size_t)PM * D * 2 /* Q hi */ + SP_KBUF * 2 * (size_t)PN * D * 2 /* K~ */ +
           2 * 2 * (size_t)D * PN * 2 /* V~^T x 2 */ + 256 /* barriers */ + 2 * PM * 4 /* row sums */;
}

// 3-input max (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (x0, x1) -> packed fp16 hi parts and lo parts with x = hi + lo to ~22 bits (hi: x with its
// mantissa truncated to fp16's 11 significant bits, exact in fp16's normal range)
__device__ __forceinline__ void split16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const float h0 = __uint_as_float(__float_as_uint(x0) & 0xFFFFE000u);
    const float h1 = __uint_as_float(__float_as_uint(x1) & 0xFFFFE000u);
    const __half2 hh = __floats2half2_rn(h0, h1);
    const __half2 ll = __floats2half2_rn(x0 - h0, x1 - h1);
    hi = *reinterpret_cast<const uint32_t*>(&hh);
    lo = *reinterpret_cast<const uint32_t*>(&ll);
}

template <int NB>
__global__ void __launch_bounds__(SP_THREADS, 1) prefill_staged(StagedArgs a) {
    constexpr int D = 32 * NB;
    constexpr int DH = D / 2;                        // O columns per owner warp
    constexpr uint32_t KT_BYTES = 2 * PN * D * 2, VT_BYTES = 2 * D * PN * 2;   // hi + lo
    const LayerView& lv = a.lv;
    extern __shared__ uint8_t raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* q_hi = sm;                              // Q hi [PM x D]; Q lo lives in TMEM
    uint8_t* kbuf = q_hi + PM * D * 2;               // SP_KBUF x (K~ hi, K~ lo)
    uint8_t* vbuf = kbuf + SP_KBUF * KT_BYTES;       // 2 x (V~^T hi, V~^T lo)
    uint64_t* bars = reinterpret_cast<uint64_t*>(vbuf + 2 * VT_BYTES);
    uint64_t* k_full = bars;                         // [SP_KBUF] K~ image landed
    uint64_t* k_empty = bars + 3;                    // [SP_KBUF] S MMAs done reading that K~ buffer
    uint64_t* v_full = bars + 6;                     // [2] V~^T image landed
    uint64_t* s_full = bars + 8;                     // S of a tile in TMEM
    uint64_t* s_empty = bars + 9;                    // owners have read it
    uint64_t* p_full = bars + 10;                    // P written to TMEM
    uint64_t* o_done = bars + 11;                    // P V~ MMAs done (P free, O readable)
    uint64_t* v_empty = bars + 12;                   // [2] P V~ MMAs done reading that V~ buffer
    volatile int* fault_flag = reinterpret_cast<volatile int*>(bars + 14);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
    float* l_part = reinterpret_cast<float*>(bars + 32);   // [2][PM] row sums of the two column halves

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool owner = warp < SP_OWNERS;
    const bool issuer = warp == SP_OWNERS && lane == 0;
    const bool copier = warp == SP_OWNERS + 1 && lane == 0;
    const bool issuer2 = warp == SP_OWNERS + 2 && lane == 0;   // the S'' MMAs
    const int hf = (warp >> 2) & 1;                  // owner column half
    const int lrow = 32 * (warp & 3) + lane;         // owner's row in the M-tile
    const int G = lv.G, H = lv.H;
    const int h = blockIdx.y, b = blockIdx.z / a.splits, sp = blockIdx.z % a.splits;
    const int rows_total = a.C * G;
    const int row0 = blockIdx.x * PM;
    const int r = row0 + lrow;
    const bool row_ok = owner && r < rows_total;
    const int ci = row_ok ? r / G : 0;
    const int gi = row_ok ? r % G : 0;
    const int n = (int)a.n;
    const int pos0 = n - a.C;
    const int my_limit = row_ok ? pos0 + ci : -1;
    const int last_row = min(rows_total - 1, row0 + PM - 1);
    const int tile_limit = pos0 + last_row / G;
    const int first_row_limit = pos0 + row0 / G;
    // this CTA's key tiles: [t_lo, t_lo + n_tiles) of the M-tile's tiles_all (every split has
    // at least one: the host splits only when the first M-tile sees splits x 32 tiles or more);
    // the loops below count tiles from t_lo
    const int tiles_all = tile_limit / PN + 1;
    const int t_lo = (int)((long long)tiles_all * sp / a.splits);
    const int n_tiles = (int)((long long)tiles_all * (sp + 1) / a.splits) - t_lo;
    const int ek = fp16_exponent(__uint_as_float(lv.stats[((long long)(b * H + h) * 2 + 0) * 2 + 1]), -120, 120);
    const int ev = fp16_exponent(__uint_as_float(lv.stats[((long long)(b * H + h) * 2 + 1) * 2 + 1]), -120, 120);
    const uint8_t* img = a.img + ((long long)(b * H + h) * a.img_tiles + t_lo) * tile_image_bytes(D);
    const long long rows_all = (long long)lv.B * a.C * G * H;
    const long long orow_idx = ((long long)b * a.C + ci) * (G * H) + (long long)h * G + gi;
    // where the row's O goes: the output row, or this split's partial
    float* const orow = a.splits > 1 ? a.part + ((long long)sp * rows_all + orow_idx) * D : a.out + orow_idx * D;

    if (tid == 0) {
        for (int i = 0; i < SP_KBUF; ++i) {
            mma::mbar_init(&k_full[i], 1);
            mma::mbar_init(&k_empty[i], 2);          // both MMA threads commit
        }
        for (int i = 0; i < 2; ++i) {
            mma::mbar_init(&v_full[i], 1);
            mma::mbar_init(&v_empty[i], 1);
        }
        mma::mbar_init(s_full, 2);                   // both MMA threads commit
        mma::mbar_init(s_empty, SP_OWNERS);
        mma::mbar_init(p_full, SP_OWNERS);
        mma::mbar_init(o_done, 1);
        *fault_flag = 0;
        mma::fence_mbar_init();
    }
    if (warp == 0) { t5::tmem_alloc(tmem_slot, 512); t5::tmem_relinquish(); }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s = tmem;                       // S': Q hi K~hi | Q hi K~lo, PN columns each
    const uint32_t t_p = tmem + 2 * PN;              // P: PN/2 columns of fp16 pairs hi, then PN/2 lo
    const uint32_t t_s3 = tmem + 3 * PN;             // S'': Q lo K~hi
    const uint32_t t_qlo = tmem + 4 * PN;            // Q lo: columns [4 PN, 4 PN + D/2)
    const uint32_t t_o = tmem + 256;                 // O: columns [256, 256 + D)
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;

    // bulk copies of a tile's K~ / V~^T images (copying thread)
    int k_last[SP_KBUF] = {-1, -1, -1}, v_last[2] = {-1, -1};
    auto copy_k = [&](int t) {
        const int kb = t % SP_KBUF;
        uint64_t* bar = &k_full[kb];
        mma::mbar_arrive_expect_tx(bar, KT_BYTES);
        mma::bulk_g2s(kbuf + (size_t)kb * KT_BYTES, img + (size_t)t * tile_image_bytes(D), KT_BYTES, bar);
        k_last[kb] = t;
    };
    auto copy_v = [&](int t) {
        uint64_t* bar = &v_full[t & 1];
        mma::mbar_arrive_expect_tx(bar, VT_BYTES);
        mma::bulk_g2s(vbuf + (size_t)(t & 1) * VT_BYTES, img + (size_t)t * tile_image_bytes(D) + KT_BYTES, VT_BYTES, bar);
        v_last[t & 1] = t;
    };
    if (copier) {
        for (int t = 0; t < SP_KBUF && t < n_tiles; ++t) copy_k(t);
        copy_v(0);
        if (n_tiles > 1) copy_v(1);
    }

    // ---- query rows: Q hi -> shared memory, Q lo -> TMEM (each owner warp of a pair writes
    // its half of the channels), normalised per row by 2^-eq; scores are multiplied back by
    // 2^(eq + ek)
    float s_mul = 1.f;
    if (owner) {
        const float* qr = a.q + (((long long)b * a.C + ci) * (G * H) + (long long)h * G + gi) * D;
        float qn = 1.f;
        if (row_ok) {
            float mq = 0.f;
            for (int c = 0; c < D; c += 4) {
                const float4 p = *reinterpret_cast<const float4*>(qr + c);
                mq = fmaxf(mq, fmaxf(fmaxf(fabsf(p.x), fabsf(p.y)), fmaxf(fabsf(p.z), fabsf(p.w))));
            }
            const int eq = fp16_exponent(mq * fabsf(a.qscale), -120, 120);
            qn = __uint_as_float((uint32_t)(127 - eq) << 23);
            s_mul = __uint_as_float((uint32_t)(127 + eq) << 23) * __uint_as_float((uint32_t)(127 + ek) << 23);
        }
#pragma unroll 1
        for (int c64 = hf * DH; c64 < (hf + 1) * DH; c64 += 64) {
            float cols[32];
#pragma unroll
            for (int k0 = 0; k0 < 64; k0 += 8) {
                float x[8], y[8];
                if (row_ok) {
                    const float4 p = *reinterpret_cast<const float4*>(qr + c64 + k0);
                    const float4 v = *reinterpret_cast<const float4*>(qr + c64 + k0 + 4);
                    x[0] = p.x; x[1] = p.y; x[2] = p.z; x[3] = p.w; x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[j] = (x[j] * a.qscale) * qn;
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[j] = 0.f;
                }
                kperm8(x, y);
                __align__(16) __half hh[8], ll[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) split16(y[j], hh[j], ll[j]);
                *reinterpret_cast<uint4*>(q_hi + t5::sw128_offset(lrow, c64 + k0, PM)) = *reinterpret_cast<const uint4*>(hh);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    cols[k0 / 2 + j] = __uint_as_float((uint32_t)__half_as_ushort(ll[2 * j]) |
                                                       ((uint32_t)__half_as_ushort(ll[2 * j + 1]) << 16));
            }
            t5::tmem_st32(t_qlo + lane_off + c64 / 2, cols);
        }
        t5::fence_proxy_async();
    }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    auto set_fault = [&]() { *fault_flag = 1; };

    float m_run = -INFINITY, l_run = 0.f;            // l_run: this warp's column half
    float gcorr = 1.f;
    int s_last = -1, o_last = -1, s2_last = -1;

    if (owner) {
        // ======================= softmax: S(t) -> P(t), running max and sum of the row
        const int oc0 = hf * DH;                     // this warp's O columns [oc0, oc0 + DH)
        for (int t = 0; t < n_tiles; ++t) {
            if (*fault_flag) break;
            const int t0 = (t_lo + t) * PN;
            if (!warp_wait(s_full, t & 1)) { set_fault(); break; }
            t5::fence_after_sync();
            float sv[32], sv2[32], sv3[32];
            t5::tmem_ld32(t_s + lane_off, sv);
            t5::tmem_ld32(t_s + PN + lane_off, sv2);
            t5::tmem_ld32(t_s3 + lane_off, sv3);
            t5::fence_before_sync();
            __syncwarp();
            if (lane == 0) mma::mbar_arrive(s_empty);
#pragma unroll
            for (int i = 0; i < PN; ++i) sv[i] += sv2[i] + sv3[i];
            if (t0 + PN - 1 > first_row_limit) {     // a tile that crosses the causal edge
#pragma unroll
                for (int i = 0; i < PN; ++i)
                    if (t0 + slot_pos(i) > my_limit) sv[i] = -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) m8[i] = fmax3(sv[4 * i], sv[4 * i + 1], fmaxf(sv[4 * i + 2], sv[4 * i + 3]));
            const float mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * s_mul;
            const bool raise = mx > m_run + PF_RESCALE || (m_run == -INFINITY && mx > -INFINITY);
            const float corr = !raise ? 1.f : ((m_run == -INFINITY) ? 0.f : mma::ex2(m_run - mx));
            if (raise) {
                l_run *= corr;
                m_run = mx;
            }
            // this warp's half of the tile: p = 2^(s * s_mul - m) (masked entries: 2^-inf = 0)
            float p[PN / 2];
#pragma unroll
            for (int j = 0; j < PN / 2; ++j) p[j] = hf ? sv[PN / 2 + j] : sv[j];
            if (m_run == -INFINITY) {
#pragma unroll
                for (int j = 0; j < PN / 2; ++j) p[j] = 0.f;
            } else {
#pragma unroll
                for (int j = 0; j < PN / 2; ++j) p[j] = mma::ex2(fmaf(p[j], s_mul, -m_run));
            }
            float ps4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) ps4[i] = (p[4 * i] + p[4 * i + 1]) + (p[4 * i + 2] + p[4 * i + 3]);
            l_run += (ps4[0] + ps4[1]) + (ps4[2] + ps4[3]);
            uint32_t ph[PN / 4], pl[PN / 4];
#pragma unroll
            for (int j = 0; j < PN / 4; ++j) split16x2(p[2 * j], p[2 * j + 1], ph[j], pl[j]);

            if (t > 0) {   // P V~(t - 1) must be done before O is rescaled and P(t) written
                if (!warp_wait(o_done, (t - 1) & 1)) { set_fault(); break; }
                t5::fence_after_sync();
            }
            if (t > 0 && t % PF_FOLD == 0) {
                // fold: O in TMEM holds tiles [t - PF_FOLD, t); add it to the partial in the
                // output row, apply this tile's correction; P V~(t) then starts afresh
                const bool first = t == PF_FOLD;
#pragma unroll 1
                for (int c = oc0; c < oc0 + DH; c += 32) {
                    float o[32];
                    t5::tmem_ld32(t_o + lane_off + c, o);
                    if (row_ok) {
#pragma unroll
                        for (int i = 0; i < 32; i += 4) {
                            float4 g4 = first ? make_float4(0.f, 0.f, 0.f, 0.f)
                                              : *reinterpret_cast<const float4*>(orow + c + i);
                            g4.x = (g4.x * gcorr + o[i]) * corr;
                            g4.y = (g4.y * gcorr + o[i + 1]) * corr;
                            g4.z = (g4.z * gcorr + o[i + 2]) * corr;
                            g4.w = (g4.w * gcorr + o[i + 3]) * corr;
                            *reinterpret_cast<float4*>(orow + c + i) = g4;
                        }
                    }
                }
                gcorr = 1.f;
            } else {
                gcorr *= corr;
                if (t > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
                    for (int c = oc0; c < oc0 + DH; c += 32) {
                        float o[32];
                        t5::tmem_ld32(t_o + lane_off + c, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= corr;
                        t5::tmem_st32(t_o + lane_off + c, o);
                    }
                }
            }
            // P hi / lo into TMEM as the A operand of the P V~ MMAs: column j < PN/2 holds the
            // fp16 hi parts of p[2j], p[2j + 1], column PN/2 + j their lo parts; this warp
            // writes columns 8 hf .. 8 hf + 7 of each
            t5::tmem_st8(t_p + lane_off + (PN / 4) * hf, ph);
            t5::tmem_st8(t_p + lane_off + PN / 2 + (PN / 4) * hf, pl);
            t5::fence_before_sync();
            __syncwarp();
            if (lane == 0) mma::mbar_arrive(p_full);
        }
    } else if (issuer) {
        // ======================= MMA issue
        // Pipe order: S(t + 1), then O(t) once P(t) is written; the softmax of tile t runs
        // while S(t + 1) executes.
        const uint32_t idesc_s2 = t5::idesc_f16(PM, 2 * PN);
        const uint32_t idesc_o = t5::idesc_f16(PM, D);
        const uint64_t dq0 = t5::desc_sw128(t5::smem_addr(q_hi));
        // buffer descriptors: the base's plus the buffer offset in the 16-byte start-address
        // field (shared-memory addresses stay below 2^18, inside the field)
        const uint64_t dk_base = t5::desc_sw128(t5::smem_addr(kbuf));
        const uint64_t dv_base = t5::desc_sw64(t5::smem_addr(vbuf));
        // S' = [Q hi K~hi | Q hi K~lo] in TMEM columns [0, 2 PN) from this thread, S'' = Q lo K~hi
        // in [3 PN, 4 PN) from the other MMA thread: the large products accumulate alone; the
        // owners add the three once both threads have committed.
        auto issue_s = [&](int t) -> bool {
            const int kb = t % SP_KBUF;
            bool okk = poll_wait(&k_full[kb], (t / SP_KBUF) & 1);
            if (okk && t >= 1) okk = poll_wait(s_empty, (t - 1) & 1);   // the owners have read S(t - 1)
            if (!okk) return false;
            t5::fence_after_sync();
            const uint64_t dk0 = dk_base + (uint64_t)((kb * KT_BYTES) >> 4);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t dq = (uint64_t)(((k >> 2) * PM * 128 + (k & 3) * 32) >> 4);
                const uint64_t dkk = (uint64_t)(((k >> 2) * 2 * PN * 128 + (k & 3) * 32) >> 4);
                t5::mma_f16_ss(t_s, dq0 + dq, dk0 + dkk, idesc_s2, k > 0);
            }
            t5::mma_commit(s_full);
            t5::mma_commit(&k_empty[kb]);
            s_last = t;
            return true;
        };
        // (no fault-flag poll in this loop: every wait is bounded and a fault ends it there)
        bool ok = issue_s(0);
        for (int t = 0; ok && t < n_tiles; ++t) {
            if (t + 1 < n_tiles) {
                ok = issue_s(t + 1);
                if (!ok) break;
            }
            ok = poll_wait(p_full, t & 1);
            if (ok) ok = poll_wait(&v_full[t & 1], (t >> 1) & 1);
            if (!ok) break;
            t5::fence_after_sync();
            const uint64_t dvh0 = dv_base + (uint64_t)(((t & 1) * VT_BYTES) >> 4);
            const uint64_t dvl0 = dvh0 + (uint64_t)((D * PN * 2) >> 4);
            // A operand (P hi / lo) from TMEM: 8 columns per 16-position k-step
#pragma unroll
            for (int k = 0; k < PN / 16; ++k) {
                const uint64_t dk = (uint64_t)((k * 32) >> 4);
                t5::mma_f16_ts(t_o, t_p + 8 * k, dvh0 + dk, idesc_o, t % PF_FOLD != 0 || k > 0);
            }
#pragma unroll
            for (int k = 0; k < PN / 16; ++k) {
                const uint64_t dk = (uint64_t)((k * 32) >> 4);
                t5::mma_f16_ts(t_o, t_p + 8 * k, dvl0 + dk, idesc_o, true);
            }
#pragma unroll
            for (int k = 0; k < PN / 16; ++k) {
                const uint64_t dk = (uint64_t)((k * 32) >> 4);
                t5::mma_f16_ts(t_o, t_p + PN / 2 + 8 * k, dvh0 + dk, idesc_o, true);
            }
            t5::mma_commit(o_done);
            t5::mma_commit(&v_empty[t & 1]);
            o_last = t;
        }
        if (!ok) set_fault();
    } else if (issuer2) {
        // ======================= the S'' MMAs of every tile, beside the other MMA thread's
        const uint32_t idesc_s = t5::idesc_f16(PM, PN);
        const uint64_t dk_base = t5::desc_sw128(t5::smem_addr(kbuf));
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            const int kb = t % SP_KBUF;
            ok = poll_wait(&k_full[kb], (t / SP_KBUF) & 1);
            if (ok && t >= 1) ok = poll_wait(s_empty, (t - 1) & 1);   // the owners have read S(t - 1)
            if (!ok) break;
            t5::fence_after_sync();
            const uint64_t dk0 = dk_base + (uint64_t)((kb * KT_BYTES) >> 4);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint64_t dkk = (uint64_t)(((k >> 2) * 2 * PN * 128 + (k & 3) * 32) >> 4);
                t5::mma_f16_ts(t_s3, t_qlo + 8 * k, dk0 + dkk, idesc_s, k > 0);
            }
            t5::mma_commit(s_full);
            t5::mma_commit(&k_empty[kb]);
            s2_last = t;
        }
        if (!ok) set_fault();
    } else if (copier) {
        // ======================= image copies: K~(t + 3) into S(t)'s buffer once S(t) has
        // finished, V~(t + 1) into O(t - 1)'s buffer once O(t - 1) has finished
        bool ok = true;
        for (int t = 0; t < n_tiles; ++t) {
            if (*fault_flag) break;
            if (t + SP_KBUF < n_tiles) {
                ok = poll_wait(&k_empty[t % SP_KBUF], (t / SP_KBUF) & 1);
                if (!ok) break;
                copy_k(t + SP_KBUF);
            }
            if (t >= 1 && t + 1 < n_tiles) {
                ok = poll_wait(&v_empty[(t - 1) & 1], ((t - 1) >> 1) & 1);
                if (!ok) break;
                copy_v(t + 1);
            }
        }
        if (!ok) set_fault();
    }

    // ---- epilogue: O / l -> out (TMEM loads by whole owner warps; only real rows store)
    if (owner) l_part[hf * PM + lrow] = l_run;
    __syncthreads();
    if (owner && !*fault_flag) {
        if (!warp_wait(o_done, (n_tiles - 1) & 1)) set_fault();
        t5::fence_after_sync();
    }
    __syncthreads();
    const bool any_fault = *fault_flag != 0;
    if (owner && !any_fault) {
        const float l_row = l_part[lrow] + l_part[PM + lrow];   // both column halves
        const float vsc = __uint_as_float((uint32_t)(127 + ev) << 23);
        // one split: O / l; several: O unnormalised, with the row's max and sum beside it
        const float inv = !row_ok ? 0.f : (a.splits > 1 ? vsc : vsc / l_row);
        if (a.splits > 1 && row_ok && hf == 0) {
            float* ml = a.part + (long long)a.splits * rows_all * D + ((long long)sp * rows_all + orow_idx) * 2;
            ml[0] = m_run;
            ml[1] = l_row;
        }
        const bool folded = n_tiles > PF_FOLD;
#pragma unroll 1
        for (int c = hf * DH; c < (hf + 1) * DH; c += 32) {
            float o[32];
            t5::tmem_ld32(t_o + lane_off + c, o);
            if (row_ok) {
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    float4 g4 = folded ? *reinterpret_cast<const float4*>(orow + c + i) : make_float4(0.f, 0.f, 0.f, 0.f);
                    g4.x = (g4.x * gcorr + o[i]) * inv;
                    g4.y = (g4.y * gcorr + o[i + 1]) * inv;
                    g4.z = (g4.z * gcorr + o[i + 2]) * inv;
                    g4.w = (g4.w * gcorr + o[i + 3]) * inv;
                    *reinterpret_cast<float4*>(orow + c + i) = g4;
                }
            }
        }
    } else if (row_ok && any_fault) {
        if (tid == 0) atomicOr(lv.status, STATUS_WAIT_TIMEOUT);
        for (int c = hf * DH; c < (hf + 1) * DH; ++c) orow[c] = __int_as_float(0x7fc00000);
    }
    // every copy issued must have landed, and every MMA finished, before the shared and
    // tensor memory are released (bounded waits; immediate on the normal path)
    if (copier) {
        for (int i = 0; i < SP_KBUF; ++i)
            if (k_last[i] >= 0) mma::mbar_wait(&k_full[i], (k_last[i] / SP_KBUF) & 1, 50000000ull);
        for (int i = 0; i < 2; ++i)
            if (v_last[i] >= 0) mma::mbar_wait(&v_full[i], (v_last[i] >> 1) & 1, 50000000ull);
    }
    if (issuer2 && s2_last >= 0) {   // this thread's last commits must land too
        mma::mbar_wait(s_full, s2_last & 1, 50000000ull);
        mma::mbar_wait(&k_empty[s2_last % SP_KBUF], (s2_last / SP_KBUF) & 1, 50000000ull);
    }
    if (issuer) {   // the later commits of each group too (their arrivals must land first)
        if (s_last >= 0) {
            mma::mbar_wait(s_full, s_last & 1, 50000000ull);
            mma::mbar_wait(&k_empty[s_last % SP_KBUF], (s_last / SP_KBUF) & 1, 50000000ull);
        }
        if (o_last >= 0) {
            mma::mbar_wait(o_done, o_last & 1, 50000000ull);
            mma::mbar_wait(&v_empty[o_last & 1], (o_last >> 1) & 1, 50000000ull);
        }
    }
    t5::fence_before_sync();
    __syncthreads();
    if (warp == 0) t5::tmem_dealloc(tmem, 512);
}

// Rows of a split prefill: out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, M = max_s m_s
// (scores in the base-2 domain). One warp per row.
__global__ void __launch_bounds__(256) prefill_merge(const float* part, float* out, long long rows_all, int splits,
                                                     int D) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows_all) return;
    const float* ml = part + (long long)splits * rows_all * D;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, ml[((long long)s * rows_all + row) * 2]);
    float L = 0.f;
    for (int s = 0; s < splits; ++s) {
        const float m = ml[((long long)s * rows_all + row) * 2];
        if (m != -INFINITY) L += mma::ex2(m - M) * ml[((long long)s * rows_all + row) * 2 + 1];
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int c = 4 * lane; c < D; c += 128) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < splits; ++s) {
            const float m = ml[((long long)s * rows_all + row) * 2];
            if (m == -INFINITY) continue;
            const float w = mma::ex2(m - M);
            const float4 o = *reinterpret_cast<const float4*>(part + ((long long)s * rows_all + row) * D + c);
            acc.x += w * o.x; acc.y += w * o.y; acc.z += w * o.z; acc.w += w * o.w;
        }
        *reinterpret_cast<float4*>(out + row * D + c) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
}

template <int NB>
cudaError_t launch_staged_nb(const StagedArgs& a, cudaStream_t st) {
    constexpr int D = 32 * NB;
    const LayerView& lv = a.lv;
    // images of every tile a row of the chunk sees: positions 0 .. n - 1
    const long long tiles = (a.n + PN - 1) / PN;
    prefill_tiles<NB><<<dim3((unsigned)tiles, (unsigned)lv.H, (unsigned)lv.B), 256, 0, st>>>(lv, a.n, (uint8_t*)a.img,
                                                                                             a.img_tiles);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    static bool raised = false;
    if (!raised) {
        e = cudaFuncSetAttribute(prefill_staged<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        raised = true;
    }
    const dim3 grid((unsigned)((a.C * lv.G + PM - 1) / PM), (unsigned)lv.H, (unsigned)(lv.B * a.splits));
    prefill_staged<NB><<<grid, SP_THREADS, sp_smem(D), st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.splits == 1) return e;
    const long long rows_all = (long long)lv.B * a.C * lv.G * lv.H;
    prefill_merge<<<(unsigned)((rows_all + 7) / 8), 256, 0, st>>>(a.part, a.out, rows_all, a.splits, D);
    return cudaGetLastError();
}

template <int NB>
cudaError_t launch_prefill_nb(PrefillArgs a, cudaStream_t st) {
    constexpr int D = 32 * NB;
    // staging halves hold PN rows of the widest row of either side and region
    int wide = 0;
    for (int kv = 0; kv < 2; ++kv) {
        wide = max(wide, a.lv.fmt[kv].stride);
        if (a.lv.W) wide = max(wide, a.lv.tail.stride);
    }
    a.stage_half = PN * wide;
    a.kbufs = pf_smem(D, 2, (size_t)a.stage_half) <= 227 * 1024 ? 2 : 1;
    const size_t smem = pf_smem(D, a.kbufs, (size_t)a.stage_half);
    static bool raised = false;
    if (!raised) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc5<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        raised = true;
    }
    const dim3 grid((unsigned)((a.C * a.lv.G + PM - 1) / PM), (unsigned)a.lv.H, (unsigned)(a.lv.B * a.splits));
    prefill_tc5<NB><<<grid, PTHREADS, smem, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.splits == 1) return e;
    const long long rows_all = (long long)a.lv.B * a.C * a.lv.G * a.lv.H;
    prefill_merge<<<(unsigned)((rows_all + 7) / 8), 256, 0, st>>>(a.part, a.out, rows_all, a.splits, D);
    return cudaGetLastError();
}

}  // namespace

bool prefill_supported(int D) { return D == 128 || D == 256; }

bool prefill_staged_used(int D, int C, int G) { return prefill_supported(D) && (long long)C * G > PM; }

size_t prefill_image_bytes(int B, int H, int D, long long max_ctx) {
    return (size_t)B * H * (size_t)((max_ctx + PN - 1) / PN) * tile_image_bytes(D);
}

size_t prefill_partial_bytes(int B, int H, int Hq, int D, int C) {
    // the staged path (several M-tiles per head) splits at most PF_MAX_SPLITS ways, the
    // on-the-fly path (one M-tile per head) at most PF_OTF_MAX_SPLITS
    const int max_splits = prefill_staged_used(D, C, Hq / H) ? PF_MAX_SPLITS : PF_OTF_MAX_SPLITS;
    return (size_t)max_splits * B * C * Hq * (D + 2) * sizeof(float);
}

// Key-range splits of the staged prefill: CTAs (one per SM) = M-tiles x H x B x splits; the
// count that fills the last wave best, each extra split charged 1% (its pipeline start and
// the merge), and only while every split of the first M-tile keeps 32 tiles or more.
int prefill_splits(int B, int H, int G, int C, long long n, int num_sms) {
    const long long ctas = (long long)((C * G + PM - 1) / PM) * H * B;
    const long long first_tiles = (n - C + (std::min(C * G, PM) - 1) / G) / PN + 1;
    int best = 1;
    double best_score = -1.0;
    for (int s = 1; s <= PF_MAX_SPLITS; ++s) {
        if (s > 1 && first_tiles < 32LL * s) break;
        const long long units = ctas * s;
        const long long waves = (units + num_sms - 1) / num_sms;
        const double score = (double)units / ((double)waves * num_sms) - 0.01 * (s - 1);
        if (score > best_score + 1e-9) { best_score = score; best = s; }
    }
    return best;
}

// Key-range splits of the on-the-fly prefill (C * G <= 128: one M-tile per head, few CTAs):
// as many as fill one wave of CTAs (one per SM), up to PF_OTF_MAX_SPLITS, while every split
// keeps 32 tiles or more.
int prefill_otf_splits(int B, int H, int G, int C, long long n, int num_sms) {
    const long long ctas = (long long)((C * G + PM - 1) / PM) * H * B;
    const long long first_tiles = (n - C + (std::min(C * G, PM) - 1) / G) / PN + 1;
    long long s = num_sms / ctas;
    s = std::min(s, first_tiles / 32);
    s = std::min(s, (long long)PF_OTF_MAX_SPLITS);
    return (int)std::max(1LL, s);
}

cudaError_t launch_prefill(const LayerView& lv, const float* q, float scale, float* out, long long n, int C,
                           cudaStream_t st, uint8_t* img, long long img_tiles, float* part, size_t part_bytes,
                           int num_sms) {
    // splits the partial area holds
    const long long per_split = (long long)lv.B * C * lv.G * lv.H * (lv.D + 2) * (long long)sizeof(float);
    const int cap = part ? (int)std::min<long long>(PF_OTF_MAX_SPLITS, (long long)(part_bytes / per_split)) : 1;
    if (img && prefill_staged_used(lv.D, C, lv.G)) {
        StagedArgs s{};
        s.lv = lv;
        s.q = q;
        s.out = out;
        s.qscale = scale * 1.4426950408889634f;
        s.n = n;
        s.C = C;
        s.img = img;
        s.img_tiles = img_tiles;
        s.splits = cap >= 2 ? std::min(cap, prefill_splits(lv.B, lv.H, lv.G, C, n, num_sms)) : 1;
        s.part = part;
        if (lv.D == 256) return launch_staged_nb<8>(s, st);
        if (lv.D == 128) return launch_staged_nb<4>(s, st);
        return cudaErrorInvalidValue;
    }
    PrefillArgs a{};
    a.lv = lv;
    a.q = q;
    a.out = out;
    a.qscale = scale * 1.4426950408889634f;
    a.n = n;
    a.C = C;
    a.splits = cap >= 2 ? std::min(cap, prefill_otf_splits(lv.B, lv.H, lv.G, C, n, num_sms)) : 1;
    a.part = part;
    if (lv.D == 256) return launch_prefill_nb<8>(a, st);
    if (lv.D == 128) return launch_prefill_nb<4>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace kvq
