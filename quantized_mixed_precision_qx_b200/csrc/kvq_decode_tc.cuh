// kvq_decode_tc.cuh -- split-K decode / row-batched prefill pass 1 on warp-level tensor
// cores, for head_dim 128 or 256 (nb = 4 or 8 blocks of 32 channels).
//
// CTA = 8 consumer warps + 1 producer warp. The producer streams the split's rows in
// 64-row tiles with 1-D bulk copies (TMA engine) into a 2-stage shared-memory ring
// (K tile and V tile are each one contiguous copy, since a region stores its rows back
// to back). A tile has 4 groups of 16 rows; each group is shared by a pair of consumer
// warps, one per half of the channel blocks:
//   S^T[16 x 8] = K[16 x D] Q^T[D x 8]   (m16n8k16; rows = tokens, 8 = the G <= 8 heads),
//       each warp of the pair summing its half of the blocks; the two halves are
//       exchanged through shared memory, so both warps hold the same S
//   p = exp2(S - m) with a per-head running max m and sum l (online softmax; computed
//       identically by both warps of the pair)
//   O^T[D/2 x 8] += V^T[D/2 x 16] P^T[16 x 8]   (each warp: the output channels of its half)
// Codes enter the MMAs exactly (fp16 integers); K block scales are applied to the QK
// accumulators per 32-channel block, V block scales are folded into the V operand as an
// exact hi + lo fp16 pair; the query and P are split into hi + lo parts. At the end the
// 4 row groups' states are merged in shared memory and the CTA writes one (m, l, o)
// partial per head, like the CUDA-core path.
#pragma once
#include "kvq_mma.cuh"

namespace kvq {
namespace tc {

constexpr int TOK = 64;                  // rows per stage
constexpr int STAGES = 2;
constexpr int TGROUPS = TOK / 16;        // 16-row groups of a tile
constexpr int CWARPS = 2 * TGROUPS;      // consumer warps: (row group, channel half)
constexpr int THREADS = 32 * (CWARPS + 1);
constexpr int NBMAX = 8;
// Lazy rescale: a head's running max is only raised when a score exceeds it by more
// than 2^8, so p stays <= 256 and the accumulators are rescaled rarely. Results are
// mathematically unchanged (m, l and o always refer to the same stale max).
constexpr float RESCALE_THRESHOLD = 8.0f;

struct Args {
    const uint8_t* kbase;   // first row of this (b, h) K region
    const uint8_t* vbase;
    int kstride, vstride;   // row strides (bytes)
    const float* q;         // [B][rows][Hq][D]
    float qscale;           // scale * log2(e)
    const float* scales;    // KVarN [B][H][2][D] or nullptr
    const uint32_t* stats;  // the layer's value bounds [B][H][2][2] (float bits)
    uint32_t* status;       // device status word (a timed-out wait is recorded here)
    float* ws;
    long long n;            // cached positions
    long long pos_base;     // position of query row 0
    int rows;
    int ring;               // region: 0 low-bit, 1 ring
    int W;
    long long chunk;        // rows per split
    long long region_rows;
    long long region_stride_k, region_stride_v;   // bytes between (b, h) regions
    int split_offset, n_split;
    int H, G, D;
    // index-gather decode: per (batch, kv head) a list of n_idx positions (splits then run
    // over list entries); entries outside this region's positions are masked out
    const int* idx;         // [B][H][n_idx] or nullptr
    int n_idx;
    long long ring_start;   // first position held in the ring (n - W; n when W == 0)
    // 0: first launch of the call (lets the next launch start early);
    // 1: launched as a programmatic dependent of the previous pass: runs concurrently
    //    with it and, before exiting, waits for it to finish, so a later dependent that
    //    waits on this grid also sees the earlier one's results
    int dependent;
};

__host__ __device__ constexpr size_t stage_bytes(int ks, int vs) { return (size_t)TOK * (ks + vs); }
// shared memory: [stages | final combine (aliased)] [P transpose] [S exchange]
//                [query fragments] [query sums] [mbarriers] [fault word]
__host__ __device__ constexpr size_t comb_bytes(int D) {
    return (size_t)(TGROUPS * 8 * 3 + 16 + TGROUPS * 8 * NBMAX + TGROUPS * 8 * D) * sizeof(float);
}
__host__ __device__ constexpr size_t main_bytes(int ks, int vs, int D) {
    return ((STAGES * stage_bytes(ks, vs) > comb_bytes(D) ? STAGES * stage_bytes(ks, vs) : comb_bytes(D)) + 127) & ~(size_t)127;
}
constexpr size_t PT_BYTES = CWARPS * 16 * 8 * sizeof(float);
constexpr size_t XS_BYTES = 2 * CWARPS * 32 * sizeof(float4);       // double-buffered S halves
__host__ __device__ constexpr int query_parts(int kf) { return kf == F_BF16 ? 3 : 2; }
__host__ __device__ constexpr size_t qs_bytes(int parts) { return (size_t)NBMAX * 2 * parts * 32 * sizeof(uint2); }
constexpr size_t QSUM_BYTES = NBMAX * 8 * sizeof(float);
constexpr size_t QEXP_BYTES = 2 * 8 * sizeof(float);     // per head: 2^-e (query scaling), 2^e (score)
__host__ __device__ constexpr size_t smem_bytes(int ks, int vs, int D, int parts) {
    return main_bytes(ks, vs, D) + PT_BYTES + XS_BYTES + qs_bytes(parts) + QSUM_BYTES + QEXP_BYTES +
           2 * STAGES * sizeof(uint64_t) + STAGES * sizeof(uint64_t) + 16;
}


// OR of `pred` over the 64 threads of a warp pair (named barrier `id`); also orders the
// pair's shared-memory accesses like bar.sync
__device__ __forceinline__ bool pair_any(int id, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, 64, p;\n selp.u32 %0, 1, 0, q;\n}"
        : "=r"(r) : "r"((uint32_t)pred), "r"(id) : "memory");
    return r != 0;
}

// CTAs per SM the register allocation is sized for: head_dim 256 keeps 2 (no spills),
// head_dim 128 fits 3
__host__ __device__ constexpr int min_ctas(int nb) { return nb == 8 ? 2 : 3; }

template <int KF, int VF, int NB>
__global__ void __launch_bounds__(THREADS, min_ctas(NB)) decode_tc(Args a) {
    using namespace mma;
    using KT = Fmt<KF>;
    using VT = Fmt<VF>;
    static_assert(KT::is_bf16 == VT::is_bf16, "K and V must use the same MMA operand type");
    static_assert(NB % 2 == 0 && NB <= CWARPS, "two channel halves; one query block per warp");
    constexpr int KP = KT::parts;            // parts of the query split
    constexpr int VP = VT::parts;            // parts of the P split
    constexpr bool VSCALED = !VT::is_float;  // block scale folded into the V operand
    constexpr int HB = NB / 2;               // blocks per channel half

    extern __shared__ __align__(128) uint8_t smem[];
    const int D = 32 * NB, G = a.G, H = a.H;
    // row strides are fixed by the formats (the host passes the same values in KS,
    // VS to size shared memory)
    constexpr int KS = KT::stride(NB), VS = VT::stride(NB);
    constexpr size_t sb = stage_bytes(KS, VS);
    constexpr size_t mb = main_bytes(KS, VS, 32 * NB);
    uint8_t* stage0 = smem;
    float* pT = reinterpret_cast<float*>(smem + mb);                                   // [CWARPS][16][8]
    float4* xs = reinterpret_cast<float4*>(smem + mb + PT_BYTES);                      // [2][CWARPS][32]
    uint2* qs = reinterpret_cast<uint2*>(smem + mb + PT_BYTES + XS_BYTES);             // [NB][2][KP][32]
    float* qsum_s = reinterpret_cast<float*>(smem + mb + PT_BYTES + XS_BYTES + qs_bytes(KP));   // [NB][8]
    float* qexp_s = qsum_s + NBMAX * 8;                                                  // [2][8]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + mb + PT_BYTES + XS_BYTES + qs_bytes(KP) + QSUM_BYTES + QEXP_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* gmask = empty + STAGES;                 // gather mode: rows of each stage that were fetched
    int* fault = reinterpret_cast<int*>(gmask + STAGES);
    const bool gather = a.idx != nullptr;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int tg = warp % TGROUPS, hf = warp / TGROUPS;     // consumer: row group, channel half
    const int h = blockIdx.y, br = blockIdx.z;
    const int b = br / a.rows, r = br % a.rows;
    const int split = blockIdx.x;
    const long long limit = a.pos_base + r;

    long long t0 = (long long)split * a.chunk;
    long long t1 = t0 + a.chunk;
    if (t1 > a.region_rows) t1 = a.region_rows;
    if (!a.ring && !gather && t1 > limit + 1) t1 = limit + 1;
    if (t1 < t0) t1 = t0;
    const int n_tiles = (int)((t1 - t0 + TOK - 1) / TOK);

    const uint8_t* kreg = a.kbase + (long long)(b * H + h) * a.region_stride_k;
    const uint8_t* vreg = a.vbase + (long long)(b * H + h) * a.region_stride_v;
    const int kvarn = a.scales != nullptr && !a.ring;
    const float* sK = kvarn ? a.scales + ((long long)(b * H + h) * 2 + 0) * D : nullptr;
    const float* sV = kvarn ? a.scales + ((long long)(b * H + h) * 2 + 1) * D : nullptr;

    // V block values enter the MMA folded as fp16 hi + lo of d * c: scale d by 2^-ev so that
    // every |d * c| of the cache (bounded by the stats the appends keep) stays below 2^15, or
    // up into fp16's normal range for tiny caches
    int ev = 0;
    if constexpr (!VT::is_float) ev = fp16_exponent(__uint_as_float(a.stats[((long long)(b * H + h) * 2 + 1) * 2]), -10, 9);
    const float vexp = __uint_as_float((uint32_t)(127 + ev) << 23);         // 2^ev
    const __half vm1 = __float2half_rn(__uint_as_float((uint32_t)(127 - ev) << 23));
    const uint32_t vmul = (uint32_t)__half_as_ushort(vm1) * 0x10001u;       // 2^-ev in both halves

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // query values of this lane's fragments (warp w builds block w), loaded first so their
    // latency overlaps the setup
    float qv[2][4];
    if (warp < NB) {
        const float* qg = a.q + ((long long)br * G * H + (long long)h * G + g) * D;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) qv[m][sl] = (g < G) ? qg[32 * warp + q_channel<KF>(t, m, sl)] : 0.f;
    }
    // Rows past the end of a partial last tile are read (and multiplied by p = 0): zero
    // them in that tile's stage so they always hold finite values. In gather mode any row of
    // a tile can be masked out: zero both stages (a masked row then holds zeros or an earlier
    // tile's fetched row).
    if (gather) {
        for (size_t i = (size_t)threadIdx.x * 16; i < STAGES * sb; i += THREADS * 16)
            *reinterpret_cast<uint4*>(stage0 + i) = make_uint4(0, 0, 0, 0);
    } else if (n_tiles > 0) {
        const int last_rows = (int)(t1 - t0 - (long long)(n_tiles - 1) * TOK);
        if (last_rows < TOK) {
            uint8_t* st = stage0 + ((n_tiles - 1) % STAGES) * sb;
            const int kz0 = last_rows * KS, kz1 = TOK * KS;
            const int vz0 = kz1 + last_rows * VS, vz1 = kz1 + TOK * VS;
            for (int i = kz0 + threadIdx.x * 16; i < kz1; i += THREADS * 16)
                *reinterpret_cast<uint4*>(st + i) = make_uint4(0, 0, 0, 0);
            for (int i = vz0 + threadIdx.x * 16; i < vz1; i += THREADS * 16)
                *reinterpret_cast<uint4*>(st + i) = make_uint4(0, 0, 0, 0);
        }
    }
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], CWARPS); }
        *fault = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // ------------------------------------------------------------ producer warp
    if (warp == CWARPS && gather) {
        // one bulk copy per listed row of this region, issued by the lane that owns the row
        // (rows lane and lane + 32 of the tile); lane 0 publishes the tile's row mask
        const int* il = a.idx + ((long long)br * H + h) * a.n_idx;
        const long long W = a.W;
        int issued = 0;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % STAGES;
            int ok = 1;
            if (it >= STAGES && lane == 0) ok = mbar_wait(&empty[s], ((it / STAGES) - 1) & 1) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0) *fault = 1;
                break;
            }
            const long long r0 = t0 + (long long)it * TOK;
            const int nrows = (int)min((long long)TOK, t1 - r0);
            long long row[2];
            bool v[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int rr = lane + 32 * k;
                v[k] = false;
                row[k] = 0;
                if (rr < nrows) {
                    const long long p = il[r0 + rr];
                    if (a.ring) {
                        v[k] = p >= 0 && p >= a.ring_start && p < a.n;
                        row[k] = v[k] ? p % W : 0;
                    } else {
                        v[k] = p >= 0 && p < a.ring_start;
                        row[k] = p;
                    }
                }
            }
            const uint32_t m0 = __ballot_sync(0xffffffffu, v[0]), m1 = __ballot_sync(0xffffffffu, v[1]);
            uint8_t* st = stage0 + s * sb;
            if (lane == 0) {
                gmask[s] = (uint64_t)m0 | ((uint64_t)m1 << 32);
                const uint32_t nv = (uint32_t)(__popc(m0) + __popc(m1));
                mbar_arrive_expect_tx(&full[s], nv * (uint32_t)(KS + VS));
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                if (v[k]) {
                    const int rr = lane + 32 * k;
                    bulk_g2s(st + (size_t)rr * KS, kreg + row[k] * KS, (uint32_t)KS, &full[s]);
                    bulk_g2s(st + (size_t)TOK * KS + (size_t)rr * VS, vreg + row[k] * VS,
                             (uint32_t)VS, &full[s]);
                }
            }
            issued = it + 1;
        }
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % STAGES + STAGES) % STAGES;
                if (issued > s && last >= 0) mbar_wait(&full[s], (last / STAGES) & 1, 50000000ull);
            }
        }
    } else if (warp == CWARPS) {
        if (lane == 0) {
            int issued = 0;
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % STAGES;
                if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1)) { *fault = 1; break; }
                const long long r0 = t0 + (long long)it * TOK;
                const int nrows = (int)min((long long)TOK, t1 - r0);
                const uint32_t kb = (uint32_t)(nrows * KS), vb = (uint32_t)(nrows * VS);
                uint8_t* st = stage0 + s * sb;
                mbar_arrive_expect_tx(&full[s], kb + vb);
                bulk_g2s(st, kreg + r0 * KS, kb, &full[s]);
                bulk_g2s(st + (size_t)TOK * KS, vreg + r0 * VS, vb, &full[s]);
                issued = it + 1;
            }
            // before the stages are reused for the final combine (or the CTA exits), every
            // copy issued must have landed: wait (bounded) for the last tile of each stage;
            // when the consumers saw every tile this returns at once
            for (int s = 0; s < STAGES; ++s) {
                const int last = issued - 1 - ((issued - 1 - s) % STAGES + STAGES) % STAGES;
                if (issued > s && last >= 0) mbar_wait(&full[s], (last / STAGES) & 1, 50000000ull);
            }
        }
    }

    // ------------------------------------------------------------ query fragments
    // (B operand of QK, head g of lane (g, t)), built while the first tiles are in flight.
    // Each head's scaled query is normalised by a power of two 2^-e (e = 0 unless it lies
    // outside the fp16-friendly range); its scores are multiplied back by 2^e.
    if (warp < CWARPS) {
        {
            const int hh = warp;                     // CWARPS == 8 heads
            float mq = 0.f;
            if (hh < G) {
                const float* qh = a.q + ((long long)br * G * H + (long long)h * G + hh) * D;
                for (int c = lane; c < D; c += 32) {
                    float x = qh[c] * a.qscale;
                    if (kvarn) x *= sK[c];
                    mq = fmaxf(mq, fabsf(x));
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, off));
            if (lane == 0) {
                const int e = fp16_exponent(mq, -100, 100);
                qexp_s[hh] = __uint_as_float((uint32_t)(127 - e) << 23);
                qexp_s[8 + hh] = __uint_as_float((uint32_t)(127 + e) << 23);
            }
            asm volatile("bar.sync 1, %0;" ::"n"(32 * CWARPS) : "memory");
        }
        if (warp < NB) {
            const float qn = qexp_s[g];
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                float v[4];
#pragma unroll
                for (int sl = 0; sl < 4; ++sl) {
                    float x = qv[m][sl] * a.qscale;
                    if (kvarn) x *= sK[32 * warp + q_channel<KF>(t, m, sl)];
                    v[sl] = x * qn;
                }
                uint32_t p01[3], p23[3];
                split_pack<KF>(v[0], v[1], p01);
                split_pack<KF>(v[2], v[3], p23);
#pragma unroll
                for (int pp = 0; pp < KP; ++pp) qs[((warp * 2 + m) * KP + pp) * 32 + lane] = make_uint2(p01[pp], p23[pp]);
            }
        }
        if constexpr (KT::asym) {
            // per-block sums of the (scaled) query channels, heads 0..7
            for (int idx = threadIdx.x; idx < NB * 8; idx += 32 * CWARPS) {
                const int bb = idx >> 3, hh = idx & 7;
                float sacc = 0.f;
                if (hh < G) {
                    const float* qh = a.q + ((long long)br * G * H + (long long)h * G + hh) * D + 32 * bb;
                    const float qn = qexp_s[hh];
                    for (int c = 0; c < 32; ++c) {
                        float x = qh[c] * a.qscale;
                        if (kvarn) x *= sK[32 * bb + c];
                        sacc += x * qn;
                    }
                }
                qsum_s[idx] = sacc;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * CWARPS) : "memory");
    }

    // ------------------------------------------------------------ consumers
    float o[HB][2][4];
    float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};
    float pm[HB];                         // asym V: sum_t p_t m_t,b for head g
#pragma unroll
    for (int j = 0; j < HB; ++j) {
        pm[j] = 0.f;
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) o[j][m][i] = 0.f;
    }

    if (warp < CWARPS) {
        float* myT = pT + warp * 128;
        const int b0 = hf * HB;                      // first block of this warp's half
        const int pair_bar = 2 + tg;                 // named barrier of the row-group pair
        // ring slot s holds position n - W + ((s + W - n mod W) mod W)
        const long long W = a.W;
        const long long nmodw = a.ring ? a.n % W : 0;
        const int sub0 = 16 * tg;
        const float qe0 = qexp_s[8 + 2 * t], qe1 = qexp_s[8 + 2 * t + 1];   // 2^e of heads 2t, 2t+1
        const bool qscaled = qe0 != 1.f || qe1 != 1.f;
        for (int it = 0; it < n_tiles; ++it) {
            const int s = it % STAGES;
            const bool ok = mbar_wait(&full[s], (it / STAGES) & 1);
            const long long r0 = t0 + (long long)it * TOK;
            const int nrows = (int)min((long long)TOK, t1 - r0);
            if (sub0 < nrows) {                      // uniform over the pair
                const uint8_t* kt = stage0 + s * sb;
                const uint8_t* vt = kt + (size_t)TOK * KS;
                const uint64_t gm = gather ? gmask[s] : 0ull;
                auto valid = [&](int rr) -> bool {
                    if (gather) return (gm >> (sub0 + rr)) & 1ull;
                    if (sub0 + rr >= nrows) return false;
                    if (a.ring) {
                        long long d = r0 + sub0 + rr + W - nmodw;
                        if (d >= W) d -= W;
                        return a.n - W + d <= limit;
                    }
                    return true;
                };
                // ---------------- S^T = K Q^T over this warp's blocks
                const uint8_t* rg = kt + (size_t)(sub0 + g) * KS;
                const uint8_t* rg8 = kt + (size_t)(sub0 + g + 8) * KS;
                float sc[4] = {0.f, 0.f, 0.f, 0.f};
                if (ok && !KT::is_float) {
                    // slot t of this warp's blocks of rows g and g + 8: one wide load per plane
                    RowPieces<KF, NB, HB> kg, kg8;
                    kg.load(rg, b0, t);
                    kg8.load(rg8, b0, t);
#pragma unroll
                    for (int j = 0; j < HB; ++j) {
                        const int bb = b0 + j;
                        uint32_t pg[4], pg8[4];
                        k_pairs_r<KF, NB, HB>(kg, j, pg);
                        k_pairs_r<KF, NB, HB>(kg8, j, pg8);
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            const uint32_t af[4] = {pg[2 * m], pg8[2 * m], pg[2 * m + 1], pg8[2 * m + 1]};
#pragma unroll
                            for (int pp = 0; pp < KP; ++pp) {
                                const uint2 qv2 = qs[((bb * 2 + m) * KP + pp) * 32 + lane];
                                mma_f<KF>(acc, af, qv2.x, qv2.y);
                            }
                        }
                        const uint32_t dsel = (j & 1) ? 0x7632u : 0x5410u;
                        const uint32_t dd = prmt(kg.d[j >> 1], kg8.d[j >> 1], dsel);
                        const float2 df = __half22float2(*reinterpret_cast<const __half2*>(&dd));
                        sc[0] = fmaf(acc[0], df.x, sc[0]);
                        sc[1] = fmaf(acc[1], df.x, sc[1]);
                        sc[2] = fmaf(acc[2], df.y, sc[2]);
                        sc[3] = fmaf(acc[3], df.y, sc[3]);
                        if constexpr (KT::asym) {
                            const uint32_t mm = prmt(kg.m[j >> 1], kg8.m[j >> 1], dsel);
                            const float2 mf = __half22float2(*reinterpret_cast<const __half2*>(&mm));
                            const float2 qq = *reinterpret_cast<const float2*>(&qsum_s[bb * 8 + 2 * t]);
                            sc[0] = fmaf(mf.x, qq.x, sc[0]);
                            sc[1] = fmaf(mf.x, qq.y, sc[1]);
                            sc[2] = fmaf(mf.y, qq.x, sc[2]);
                            sc[3] = fmaf(mf.y, qq.y, sc[3]);
                        }
                    }
                } else if (ok) {
#pragma unroll
                    for (int j = 0; j < HB; ++j) {
                        const int bb = b0 + j;
                        uint32_t af[2][4];
                        k_frags<KF>(rg, rg8, NB, bb, t, af);
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int m = 0; m < 2; ++m)
#pragma unroll
                            for (int pp = 0; pp < KP; ++pp) {
                                const uint2 qv2 = qs[((bb * 2 + m) * KP + pp) * 32 + lane];
                                mma_f<KF>(acc, af[m], qv2.x, qv2.y);
                            }
                        if constexpr (KT::is_float) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) sc[i] += acc[i];
                        } else {
                            const float dg = h2f_lo(reinterpret_cast<const uint16_t*>(rg)[bb]);
                            const float dg8 = h2f_lo(reinterpret_cast<const uint16_t*>(rg8)[bb]);
                            sc[0] = fmaf(acc[0], dg, sc[0]);
                            sc[1] = fmaf(acc[1], dg, sc[1]);
                            sc[2] = fmaf(acc[2], dg8, sc[2]);
                            sc[3] = fmaf(acc[3], dg8, sc[3]);
                            if constexpr (KT::asym) {
                                const float mg = h2f_lo(reinterpret_cast<const uint16_t*>(rg + KT::off_m(NB))[bb]);
                                const float mg8 = h2f_lo(reinterpret_cast<const uint16_t*>(rg8 + KT::off_m(NB))[bb]);
                                const float2 qq = *reinterpret_cast<const float2*>(&qsum_s[bb * 8 + 2 * t]);
                                sc[0] = fmaf(mg, qq.x, sc[0]);
                                sc[1] = fmaf(mg, qq.y, sc[1]);
                                sc[2] = fmaf(mg8, qq.x, sc[2]);
                                sc[3] = fmaf(mg8, qq.y, sc[3]);
                            }
                        }
                    }
                }
                // ---------------- exchange the halves (and any wait failure) within the pair
                float4* xb = xs + (it & 1) * CWARPS * 32;
                xb[warp * 32 + lane] = make_float4(sc[0], sc[1], sc[2], sc[3]);
                if (pair_any(pair_bar, !ok)) { *fault = 1; break; }
                {
                    const float4 ps = xb[(warp ^ TGROUPS) * 32 + lane];
                    sc[0] += ps.x; sc[1] += ps.y; sc[2] += ps.z; sc[3] += ps.w;   // commutative: same in both
                }
                if (qscaled) { sc[0] *= qe0; sc[1] *= qe1; sc[2] *= qe0; sc[3] *= qe1; }
                if (!valid(g)) { sc[0] = -INFINITY; sc[1] = -INFINITY; }
                if (!valid(g + 8)) { sc[2] = -INFINITY; sc[3] = -INFINITY; }
                // ---------------- online softmax for heads 2t, 2t+1
                float mx0 = fmaxf(sc[0], sc[2]), mx1 = fmaxf(sc[1], sc[3]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const bool up0 = mx0 > mrun[0] + RESCALE_THRESHOLD || (mrun[0] == -INFINITY && mx0 > -INFINITY);
                const bool up1 = mx1 > mrun[1] + RESCALE_THRESHOLD || (mrun[1] == -INFINITY && mx1 > -INFINITY);
                if (__any_sync(0xffffffffu, up0 || up1)) {
                    const float mn0 = up0 ? mx0 : mrun[0];
                    const float mn1 = up1 ? mx1 : mrun[1];
                    const float c0 = (mrun[0] == -INFINITY) ? 0.f : ex2(mrun[0] - mn0);
                    const float c1 = (mrun[1] == -INFINITY) ? 0.f : ex2(mrun[1] - mn1);
                    lrun[0] *= c0;
                    lrun[1] *= c1;
#pragma unroll
                    for (int j = 0; j < HB; ++j)
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            o[j][m][0] *= c0; o[j][m][1] *= c1;
                            o[j][m][2] *= c0; o[j][m][3] *= c1;
                        }
                    if constexpr (VT::asym) {
                        // pm belongs to head g: fetch that head's factor from lane (g >> 1)
                        const float f0 = __shfl_sync(0xffffffffu, c0, g >> 1);
                        const float f1 = __shfl_sync(0xffffffffu, c1, g >> 1);
                        const float cg = (g & 1) ? f1 : f0;
#pragma unroll
                        for (int j = 0; j < HB; ++j) pm[j] *= cg;
                    }
                    mrun[0] = mn0;
                    mrun[1] = mn1;
                }
                float p[4];
                if (mrun[0] == -INFINITY) { p[0] = 0.f; p[2] = 0.f; }
                else { p[0] = ex2(sc[0] - mrun[0]); p[2] = ex2(sc[2] - mrun[0]); }
                if (mrun[1] == -INFINITY) { p[1] = 0.f; p[3] = 0.f; }
                else { p[1] = ex2(sc[1] - mrun[1]); p[3] = ex2(sc[3] - mrun[1]); }
                lrun[0] += p[0] + p[2];
                lrun[1] += p[1] + p[3];
                // ---------------- transpose P: (tokens g, g+8; heads 2t, 2t+1) -> (tokens 2t.., head g)
                *reinterpret_cast<float2*>(&myT[g * 8 + 2 * t]) = make_float2(p[0], p[1]);
                *reinterpret_cast<float2*>(&myT[(g + 8) * 8 + 2 * t]) = make_float2(p[2], p[3]);
                __syncwarp();
                const int tk0 = 2 * t, tk2 = 2 * t + 8;
                float pv[4];
                pv[0] = myT[tk0 * 8 + g];
                pv[1] = myT[(tk0 + 1) * 8 + g];
                pv[2] = myT[tk2 * 8 + g];
                pv[3] = myT[(tk2 + 1) * 8 + g];
                __syncwarp();
                const bool v0 = valid(tk0), v1 = valid(tk0 + 1), v2 = valid(tk2), v3 = valid(tk2 + 1);
                const uint8_t* vr0 = vt + (size_t)(sub0 + tk0) * VS;
                const uint8_t* vr1 = vr0 + VS;
                const uint8_t* vr2 = vt + (size_t)(sub0 + tk2) * VS;
                const uint8_t* vr3 = vr2 + VS;
                // P split once per sub-tile (invalid tokens carry p = 0)
                uint32_t bp[3][2];
                {
                    uint32_t x01[3], x23[3];
                    split_pack<VF>(v0 ? pv[0] : 0.f, v1 ? pv[1] : 0.f, x01);
                    split_pack<VF>(v2 ? pv[2] : 0.f, v3 ? pv[3] : 0.f, x23);
#pragma unroll
                    for (int pp = 0; pp < 3; ++pp) { bp[pp][0] = x01[pp]; bp[pp][1] = x23[pp]; }
                }
                // ---------------- O^T += V^T P^T over this warp's blocks
                // slot g >> 1 of this warp's blocks of the four rows: one wide load per plane
                RowPieces<VF, NB, HB> vp0, vp1, vp2, vp3;
                if constexpr (VSCALED) {
                    vp0.load(vr0, b0, g >> 1);
                    vp1.load(vr1, b0, g >> 1);
                    vp2.load(vr2, b0, g >> 1);
                    vp3.load(vr3, b0, g >> 1);
                }
#pragma unroll
                for (int j = 0; j < HB; ++j) {
                    const int bb = b0 + j;
                    if constexpr (VSCALED) {
                        uint32_t ah[2][4], al[2][4];
                        v_frags_scaled_r<VF, NB, HB>(vp0, vp1, vp2, vp3, j, g & 1, vmul, ah, al);
#pragma unroll
                        for (int m = 0; m < 2; ++m) {
                            mma_f16(o[j][m], ah[m], bp[0][0], bp[0][1]);
                            mma_f16(o[j][m], ah[m], bp[1][0], bp[1][1]);
                            mma_f16(o[j][m], al[m], bp[0][0], bp[0][1]);
                        }
                        if constexpr (VT::asym) {
                            // min term of the centred codes: m + d * c (c = (2^bits - 1)/2)
                            constexpr float VC = VT::vcenter;
                            const uint32_t dsel = (j & 1) ? 0x7632u : 0x5410u;
                            const uint32_t d01 = prmt(vp0.d[j >> 1], vp1.d[j >> 1], dsel);
                            const uint32_t d23 = prmt(vp2.d[j >> 1], vp3.d[j >> 1], dsel);
                            const uint32_t m01 = prmt(vp0.m[j >> 1], vp1.m[j >> 1], dsel);
                            const uint32_t m23 = prmt(vp2.m[j >> 1], vp3.m[j >> 1], dsel);
                            const float2 fd01 = __half22float2(*reinterpret_cast<const __half2*>(&d01));
                            const float2 fd23 = __half22float2(*reinterpret_cast<const __half2*>(&d23));
                            const float2 fm01 = __half22float2(*reinterpret_cast<const __half2*>(&m01));
                            const float2 fm23 = __half22float2(*reinterpret_cast<const __half2*>(&m23));
                            const float m0 = fmaf(fd01.x, VC, fm01.x);
                            const float m1 = fmaf(fd01.y, VC, fm01.y);
                            const float m2 = fmaf(fd23.x, VC, fm23.x);
                            const float m3 = fmaf(fd23.y, VC, fm23.y);
                            float acc = pm[j];
                            if (v0) acc = fmaf(pv[0], m0, acc);
                            if (v1) acc = fmaf(pv[1], m1, acc);
                            if (v2) acc = fmaf(pv[2], m2, acc);
                            if (v3) acc = fmaf(pv[3], m3, acc);
                            pm[j] = acc;
                        }
                    } else {
                        uint32_t af[2][4];
                        v_frags<VF>(vr0, vr1, vr2, vr3, NB, bb, g, af);
#pragma unroll
                        for (int m = 0; m < 2; ++m)
#pragma unroll
                            for (int pp = 0; pp < VP; ++pp) mma_f<VF>(o[j][m], af[m], bp[pp][0], bp[pp][1]);
                    }
                }
            } else if (!ok) {
                *fault = 1;
                break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }

    // ------------------------------------------------------------ combine the 4 row groups
    __syncthreads();
    // shared layout (reusing the stages): cm[TGROUPS][8], cl[TGROUPS][8],
    // cpm[TGROUPS][8][NBMAX], co[TGROUPS][8][D]
    float* cm = reinterpret_cast<float*>(smem);
    float* cl = cm + TGROUPS * 8;
    float* cpm = cl + TGROUPS * 8;
    float* co = cpm + TGROUPS * 8 * NBMAX;
    if (warp < CWARPS) {
        const int b0 = hf * HB;
        if (hf == 0) {
            // l: reduce the per-thread partial sums over the 8 lanes sharing t (the pair
            // holds identical m and l)
            float l0 = lrun[0], l1 = lrun[1];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                l1 += __shfl_xor_sync(0xffffffffu, l1, off);
            }
            if (g == 0) {
                cm[tg * 8 + 2 * t] = mrun[0];
                cm[tg * 8 + 2 * t + 1] = mrun[1];
                cl[tg * 8 + 2 * t] = l0;
                cl[tg * 8 + 2 * t + 1] = l1;
            }
        }
        if constexpr (VT::asym) {
#pragma unroll
            for (int j = 0; j < HB; ++j) {
                float v = pm[j];
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                if (t == 0) cpm[(tg * 8 + g) * NBMAX + b0 + j] = v;
            }
        }
#pragma unroll
        for (int j = 0; j < HB; ++j) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int c_lo = 32 * (b0 + j) + v_channel(g, m, 0), c_hi = 32 * (b0 + j) + v_channel(g, m, 1);
                co[(tg * 8 + 2 * t) * D + c_lo] = o[j][m][0];
                co[(tg * 8 + 2 * t + 1) * D + c_lo] = o[j][m][1];
                co[(tg * 8 + 2 * t) * D + c_hi] = o[j][m][2];
                co[(tg * 8 + 2 * t + 1) * D + c_hi] = o[j][m][3];
            }
        }
    }
    __syncthreads();
    // per head: max over the row groups, each group's weight and the weighted sum of l
    float* cw = co + TGROUPS * 8 * D;     // [TGROUPS][8]
    float* cM = cw + TGROUPS * 8;         // [8]
    float* cL = cM + 8;                   // [8]
    const bool bad = *fault != 0;
    if (threadIdx.x < 8) {
        const int hh = threadIdx.x;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < TGROUPS; ++w) M = fmaxf(M, cm[w * 8 + hh]);
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < TGROUPS; ++w) {
            const float mw = cm[w * 8 + hh];
            const float e = (M == -INFINITY || mw == -INFINITY) ? 0.f : ex2(mw - M);
            cw[w * 8 + hh] = e;
            L = fmaf(cl[w * 8 + hh], e, L);
        }
        cM[hh] = M;
        cL[hh] = bad ? __int_as_float(0x7fc00000) : L;   // a timed-out wait poisons the result
    }
    if (bad && threadIdx.x == 0) atomicOr(a.status, STATUS_WAIT_TIMEOUT);
    __syncthreads();
    float* part = a.ws + ((((long long)br * H + h) * a.n_split) + a.split_offset + split) * ((long long)G * (D + 2));
    // o = sum over row groups of weight * o_w, two channels per thread step (8-byte stores)
    for (int idx = 2 * threadIdx.x; idx < G * D; idx += 2 * THREADS) {
        const int hh = idx / D, c = idx % D;
        float o0 = 0.f, o1 = 0.f;
#pragma unroll
        for (int w = 0; w < TGROUPS; ++w) {
            const float e = cw[w * 8 + hh];
            float2 ow = *reinterpret_cast<const float2*>(&co[(w * 8 + hh) * D + c]);
            if constexpr (VT::asym) {
                const float pmw = cpm[(w * 8 + hh) * NBMAX + (c >> 5)];
                ow.x = fmaf(ow.x, vexp, pmw);
                ow.y = fmaf(ow.y, vexp, pmw);
            } else if constexpr (VSCALED) {
                ow.x *= vexp;
                ow.y *= vexp;
            }
            o0 = fmaf(ow.x, e, o0);
            o1 = fmaf(ow.y, e, o1);
        }
        if (sV) { o0 *= sV[c]; o1 *= sV[c + 1]; }
        *reinterpret_cast<float2*>(&part[2 * G + idx]) = make_float2(o0, o1);
    }
    if (threadIdx.x < G) {
        part[threadIdx.x] = cM[threadIdx.x];
        part[G + threadIdx.x] = cL[threadIdx.x];
    }
    if (a.dependent) asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace tc
}  // namespace kvq
