// kvq_prefill.cu -- causal chunked-prefill attention on 5th-generation tensor cores.
//
// The chunk's C rows were just appended at positions n - C .. n - 1; chunk row i attends
// to positions t <= n - C + i of the post-append cache (low-bit rows below the window,
// ring rows inside it). QK^T and PV are dense contractions, so they run as tcgen05 MMAs
// with fp32 accumulators in tensor memory:
//
//   CTA   = 128 query rows of one (batch, kv head): row r = chunk row * G + head in group,
//           TMEM lane r; 4 warps, one thread per row.
//   tile  = 64 key positions. Each tile is dequantized into shared memory as exact fp16
//           hi + lo parts (K~ = hi + lo; the query and P are split the same way), and
//           S = Qh Kh^T + Qh Kl^T + Ql Kh^T (3 passes, M128 N64 K16 steps) -> TMEM cols [0, 64)
//           O += Ph Vh + Ph Vl + Pl Vh    (3 passes, M128 N256 K16 steps) -> TMEM cols [256, 512)
//   The softmax is row-local (each thread owns its row), with a lazily raised running max.
//
// Shared memory (head_dim D = 32 NB): Q hi/lo 2 x 128 x D x 2 B, a K/V tile buffer
// 2 x 64 x D x 2 B (K~ first, then V~^T), P hi/lo 2 x 128 x 64 x 2 B. All operands use the
// K-major 128-byte-swizzled layout of kvq_tc5.cuh.
#include "kvq_internal.cuh"
#include "kvq_mma.cuh"
#include "kvq_tc5.cuh"

namespace kvq {
namespace {

constexpr int PM = 128;           // query rows per CTA
constexpr int PN = 64;            // key positions per tile
constexpr int PTHREADS = 128;
constexpr float PF_RESCALE = 8.0f;

struct PrefillArgs {
    LayerView lv;
    const float* q;               // [B][C][Hq][D]
    float* out;                   // [B][C][Hq][D]
    float qscale;                 // scale * log2(e)
    long long n;                  // cached positions (after the append)
    int C;                        // chunk rows
    int* fault;                   // optional device fault word (may be null)
};

__host__ __device__ constexpr size_t pf_smem(int D) {
    return 1024 /* alignment slack */ + 2 * (size_t)PM * D * 2 + 2 * (size_t)PN * D * 2 + 2 * (size_t)PM * PN * 2 + 64;
}

// value of channel c0 + j (j < 8) of a stored row; c0 % 8 == 0
__device__ __forceinline__ void decode8(const uint8_t* __restrict__ row, const RowFmt& f, int c0, float (&x)[8]) {
    if (f.kind != 0) {
        const uint4 w = *reinterpret_cast<const uint4*>(row + 2 * c0);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (f.kind == 1) {
                x[2 * j] = __uint_as_float(ws[j] << 16);
                x[2 * j + 1] = __uint_as_float(ws[j] & 0xFFFF0000u);
            } else {
                x[2 * j] = mma::h2f_lo(ws[j]);
                x[2 * j + 1] = mma::h2f_hi(ws[j]);
            }
        }
        return;
    }
    const int blk = c0 >> 5;
    const float d = mma::h2f_lo(reinterpret_cast<const uint16_t*>(row)[blk]);
    const float m = f.asym ? mma::h2f_lo(reinterpret_cast<const uint16_t*>(row + f.off_m)[blk]) : 0.f;
    uint64_t p0;
    const uint8_t* a0 = row + f.off_p0 + c0 * f.w0 / 8;
    if (f.w0 == 8) p0 = *reinterpret_cast<const unsigned long long*>(a0);
    else if (f.w0 == 4) p0 = *reinterpret_cast<const uint32_t*>(a0);
    else p0 = *reinterpret_cast<const uint16_t*>(a0);
    uint32_t p1 = 0;
    if (f.w1 == 2) p1 = *reinterpret_cast<const uint16_t*>(row + f.off_p1 + c0 / 4);
    else if (f.w1 == 1) p1 = row[f.off_p1 + c0 / 8];
    const uint32_t m0 = (1u << f.w0) - 1, m1 = (1u << f.w1) - 1;
    const int off = 1 << (f.bits - 1);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int u = (int)(((uint32_t)(p0 >> (j * f.w0)) & m0) | (((p1 >> (j * f.w1)) & m1) << f.w0));
        x[j] = f.asym ? __fadd_rn(__fmul_rn(d, (float)u), m) : __fmul_rn(d, (float)(u - off));
    }
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

// stored row of position t (low-bit store or ring) and whether KVarN scales apply
__device__ __forceinline__ const uint8_t* position_row(const LayerView& lv, int b, int h, int kv, long long t,
                                                       long long n, const RowFmt*& f, const float*& s) {
    const long long W = lv.W;
    if (W > 0 && t >= n - W) {
        f = &lv.tail;
        s = nullptr;
        return lv.ring[kv] + (long long)(b * lv.H + h) * lv.ring_region + (t % W) * lv.tail.stride;
    }
    f = &lv.fmt[kv];
    s = lv.kvarn ? lv.scales + ((long long)(b * lv.H + h) * 2 + kv) * lv.D : nullptr;
    return lv.main[kv] + (long long)(b * lv.H + h) * lv.main_region[kv] + t * lv.fmt[kv].stride;
}

template <int NB>
__global__ void __launch_bounds__(PTHREADS, 1) prefill_tc5(PrefillArgs a) {
    constexpr int D = 32 * NB;
    const LayerView& lv = a.lv;
    extern __shared__ uint8_t raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* q_hi = sm;
    uint8_t* q_lo = q_hi + PM * D * 2;
    uint8_t* kv_hi = q_lo + PM * D * 2;              // K~ [PN x D], later V~^T [D x PN]
    uint8_t* kv_lo = kv_hi + PN * D * 2;
    uint8_t* p_hi = kv_lo + PN * D * 2;              // P [PM x PN]
    uint8_t* p_lo = p_hi + PM * PN * 2;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(p_lo + PM * PN * 2);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 1);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int G = lv.G, H = lv.H;
    const int h = blockIdx.y, b = blockIdx.z;
    const int rows_total = a.C * G;
    const int r = blockIdx.x * PM + tid;             // query row of this thread
    const bool row_ok = r < rows_total;
    const int ci = row_ok ? r / G : 0;               // chunk row
    const int gi = row_ok ? r % G : 0;
    const long long pos0 = a.n - a.C;
    const long long my_limit = row_ok ? pos0 + ci : -1;   // last visible position
    const int last_row = min(rows_total - 1, (int)blockIdx.x * PM + PM - 1);
    const long long tile_limit = pos0 + last_row / G;      // last position any row sees
    const long long first_row_limit = pos0 + ((int)blockIdx.x * PM) / G;

    // ---- query rows -> Q hi/lo (scaled to base-2 logits)
    {
        const float* qr = a.q + (((long long)b * a.C + ci) * (G * H) + (long long)h * G + gi) * D;
#pragma unroll 1
        for (int k0 = 0; k0 < D; k0 += 8) {
            float x[8];
            if (row_ok) {
                const float4 u = *reinterpret_cast<const float4*>(qr + k0);
                const float4 v = *reinterpret_cast<const float4*>(qr + k0 + 4);
                x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w; x[4] = v.x; x[5] = v.y; x[6] = v.z; x[7] = v.w;
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] *= a.qscale;
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = 0.f;
            }
            store_chunk(q_hi, q_lo, tid, k0, PM, x);
        }
    }
    if (tid == 0) { mma::mbar_init(mbar, 1); mma::fence_mbar_init(); }
    if (warp == 0) { t5::tmem_alloc(tmem_slot, 512); t5::tmem_relinquish(); }
    t5::fence_before_sync();
    __syncthreads();
    t5::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s = tmem;                       // S: columns [0, 64)
    const uint32_t t_o = tmem + 256;                 // O: columns [256, 512)
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

    const uint32_t idesc_s = t5::idesc_f16(PM, PN);
    const uint32_t idesc_o = t5::idesc_f16(PM, D);
    const uint32_t sq_hi = t5::smem_addr(q_hi), sq_lo = t5::smem_addr(q_lo);
    const uint32_t skv_hi = t5::smem_addr(kv_hi), skv_lo = t5::smem_addr(kv_lo);
    const uint32_t sp_hi = t5::smem_addr(p_hi), sp_lo = t5::smem_addr(p_lo);

    float m_run = -INFINITY, l_run = 0.f;
    uint32_t phase = 0;
    bool have_o = false;
    bool fault = false;
    const long long n_tiles = tile_limit / PN + 1;

    for (long long tile = 0; tile < n_tiles && !fault; ++tile) {
        const long long t0 = tile * PN;
        // ---------------- K~ tile -> hi/lo (rows = positions, k = channels); thread: half a row
        {
            const int tok = tid >> 1, half = tid & 1;
            const long long t = t0 + tok;
            const RowFmt* f;
            const float* s;
            const bool live = t <= tile_limit && t < a.n;
            const uint8_t* row = live ? position_row(lv, b, h, 0, t, a.n, f, s) : nullptr;
#pragma unroll 1
            for (int c0 = half * (D / 2); c0 < (half + 1) * (D / 2); c0 += 8) {
                float x[8];
                if (live) {
                    decode8(row, *f, c0, x);
                    if (s) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) x[j] = __fmul_rn(s[c0 + j], x[j]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) x[j] = 0.f;
                }
                store_chunk(kv_hi, kv_lo, tok, c0, PN, x);
            }
        }
        t5::fence_proxy_async();
        t5::fence_before_sync();
        __syncthreads();
        t5::fence_after_sync();
        // ---------------- S = Q K~^T (3 passes)
        if (tid == 0) {
            int step = 0;
#pragma unroll 1
            for (int pass = 0; pass < 3; ++pass) {
                const uint32_t qa = (pass == 2) ? sq_lo : sq_hi;
                const uint32_t kb = (pass == 1) ? skv_lo : skv_hi;
#pragma unroll 1
                for (int k = 0; k < D / 16; ++k, ++step) {
                    const uint64_t ad = t5::desc_sw128(qa + (k >> 2) * PM * 128 + (k & 3) * 32);
                    const uint64_t bd = t5::desc_sw128(kb + (k >> 2) * PN * 128 + (k & 3) * 32);
                    t5::mma_f16_ss(t_s, ad, bd, idesc_s, step > 0);
                }
            }
            t5::mma_commit(mbar);
        }
        fault = __syncthreads_or((!mma::mbar_wait(mbar, phase & 1)) || fault) != 0;   // uniform
        ++phase;
        t5::fence_after_sync();
        // ---------------- V~ tile -> V~^T hi/lo (rows = channels, k = positions)
        {
            // thread: 8 positions x (D/16) channel chunks of 8 -> writes whole 16-byte chunks
            const int tg = tid & 7;                  // position group: positions 8tg .. 8tg+7
            const int cg = tid >> 3;                 // channel groups cg, cg+16, ...
            const RowFmt* fr[8];
            const float* sr[8];
            const uint8_t* rowp[8];
            bool live[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const long long t = t0 + 8 * tg + j;
                live[j] = t <= tile_limit && t < a.n;
                rowp[j] = live[j] ? position_row(lv, b, h, 1, t, a.n, fr[j], sr[j]) : nullptr;
            }
#pragma unroll 1
            for (int cc = cg; cc < D / 8; cc += 16) {
                float x[8][8];                       // [position][channel]
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (live[j]) {
                        decode8(rowp[j], *fr[j], 8 * cc, x[j]);
                        if (sr[j]) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) x[j][e] = __fmul_rn(sr[j][8 * cc + e], x[j][e]);
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) x[j][e] = 0.f;
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float y[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) y[j] = x[j][e];
                    store_chunk(kv_hi, kv_lo, 8 * cc + e, 8 * tg, D, y);
                }
            }
        }
        // ---------------- softmax on S (row-local)
        {
            float sv[PN];
            float tmp[32];
            t5::tmem_ld32(t_s + lane_off, tmp);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[i] = tmp[i];
            t5::tmem_ld32(t_s + lane_off + 32, tmp);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[32 + i] = tmp[i];
            float mx = -INFINITY;
            const bool full = t0 + PN - 1 <= first_row_limit && t0 + PN <= a.n;
#pragma unroll
            for (int i = 0; i < PN; ++i) {
                if (!full && t0 + i > my_limit) sv[i] = -INFINITY;
                mx = fmaxf(mx, sv[i]);
            }
            const bool raise = mx > m_run + PF_RESCALE || (m_run == -INFINITY && mx > -INFINITY);
            const float corr = !raise ? 1.f : ((m_run == -INFINITY) ? 0.f : mma::ex2(m_run - mx));
            if (raise) {
                l_run *= corr;
                m_run = mx;
            }
            // TMEM loads/stores are warp-collective: rescale O when any lane of the warp
            // raised its max (lanes that did not use factor 1)
            if (have_o && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
                for (int c = 0; c < D; c += 32) {
                    float o[32];
                    t5::tmem_ld32(t_o + lane_off + c, o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= corr;
                    t5::tmem_st32(t_o + lane_off + c, o);
                }
            }
            float ps = 0.f;
#pragma unroll
            for (int i = 0; i < PN; ++i) {
                const float p = (m_run == -INFINITY) ? 0.f : mma::ex2(sv[i] - m_run);
                sv[i] = p;
                ps += p;
            }
            l_run += ps;
#pragma unroll
            for (int k0 = 0; k0 < PN; k0 += 8) {
                float x[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = sv[k0 + j];
                store_chunk(p_hi, p_lo, tid, k0, PM, x);
            }
        }
        t5::fence_proxy_async();
        t5::fence_before_sync();
        __syncthreads();
        t5::fence_after_sync();
        // ---------------- O += P V~ (3 passes)
        if (tid == 0) {
            int step = 0;
#pragma unroll 1
            for (int pass = 0; pass < 3; ++pass) {
                const uint32_t pa = (pass == 2) ? sp_lo : sp_hi;
                const uint32_t vb = (pass == 1) ? skv_lo : skv_hi;
#pragma unroll 1
                for (int k = 0; k < PN / 16; ++k, ++step) {
                    const uint64_t ad = t5::desc_sw128(pa + (k & 3) * 32);
                    const uint64_t bd = t5::desc_sw128(vb + (k & 3) * 32);
                    t5::mma_f16_ss(t_o, ad, bd, idesc_o, have_o || step > 0);
                }
            }
            t5::mma_commit(mbar);
        }
        fault = __syncthreads_or((!mma::mbar_wait(mbar, phase & 1)) || fault) != 0;   // uniform
        ++phase;
        have_o = true;
        t5::fence_after_sync();
    }

    // ---- epilogue: O / l -> out (TMEM loads by whole warps; only real rows store)
    const bool any_fault = __syncthreads_or(fault ? 1 : 0) != 0;
    if (have_o && !any_fault) {
        float* orow = a.out + (((long long)b * a.C + ci) * (G * H) + (long long)h * G + gi) * D;
        const float inv = row_ok ? 1.f / l_run : 0.f;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
            float o[32];
            t5::tmem_ld32(t_o + lane_off + c, o);
            if (row_ok) {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                    *reinterpret_cast<float4*>(orow + c + i) =
                        make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
            }
        }
    } else if (row_ok && any_fault) {
        float* orow = a.out + (((long long)b * a.C + ci) * (G * H) + (long long)h * G + gi) * D;
        for (int c = 0; c < D; ++c) orow[c] = __int_as_float(0x7fc00000);
    }
    t5::fence_before_sync();
    __syncthreads();
    if (warp == 0) t5::tmem_dealloc(tmem, 512);
}

template <int NB>
cudaError_t launch_prefill_nb(const PrefillArgs& a, cudaStream_t st) {
    static bool raised = false;
    const size_t smem = pf_smem(32 * NB);
    if (!raised) {
        cudaError_t e = cudaFuncSetAttribute(prefill_tc5<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        raised = true;
    }
    const dim3 grid((unsigned)((a.C * a.lv.G + PM - 1) / PM), (unsigned)a.lv.H, (unsigned)a.lv.B);
    prefill_tc5<NB><<<grid, PTHREADS, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool prefill_supported(int D) { return D == 128 || D == 256; }

cudaError_t launch_prefill(const LayerView& lv, const float* q, float scale, float* out, long long n, int C,
                           cudaStream_t st) {
    PrefillArgs a{};
    a.lv = lv;
    a.q = q;
    a.out = out;
    a.qscale = scale * 1.4426950408889634f;
    a.n = n;
    a.C = C;
    a.fault = nullptr;
    if (lv.D == 256) return launch_prefill_nb<8>(a, st);
    if (lv.D == 128) return launch_prefill_nb<4>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace kvq
