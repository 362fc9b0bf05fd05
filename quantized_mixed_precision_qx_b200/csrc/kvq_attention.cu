// kvq_attention.cu -- split-K flash-decoding over the quantized cache (decode, and the
// row-batched form used for chunked prefill), plus the fixed-order merge.
//
// Decode reads every cached byte once per step, so it is bound by HBM bytes ([OFFLOAD]:
// each decode step streams the whole attention state; the bytes read per step set the
// token rate). Pass 1: one CTA per (split, kv head, batch x query row) streams its rows,
// dequantizes in registers, and keeps an online softmax (running max m, sum l, output
// accumulator o) for the G query heads that share the KV head. Low-bit rows and ring
// rows are separate launches over separate split ranges. Pass 2 merges the splits in a
// fixed order, so results are bit-reproducible run to run.
//
// Scores are kept in base-2 units: q is pre-multiplied by scale * log2(e), so
// p = exp2(s - m) equals exp(scale * q.k - max).
#include "kvq_rowio.cuh"
#include "kvq_tc_launch.cuh"

#include <cfloat>

namespace kvq {
namespace {

constexpr int P1_WARPS = 4;
constexpr int MAXG = 8;
constexpr float LOG2E = 1.4426950408889634f;

struct P1Args {
    LayerView lv;
    const float* q;        // [B][rows][Hq][D]
    float qscale;          // scale * log2(e)
    float* ws;             // partials
    long long n;           // cached positions
    long long pos_base;    // position of query row 0
    int rows;
    int ring;              // 0: low-bit rows, 1: ring rows
    long long chunk;       // rows per split of this region
    long long region_rows; // rows of this region (n_main or n_ring)
    int split_offset;      // first split index of this region
    int n_split;           // total splits per (b, row, h)
    const int* idx;        // index-gather decode: [B][H][n_idx] positions, or nullptr
    int n_idx;
};

// Per-channel K: this lane's CPL values of the K row at position pos (pos < entered, the
// positions that have entered the K store): from the group blocks when pos's group is
// complete, else from the pending float32 row. Dequantization as for a per-token block:
// d * (u - 2^(X-1)) or d * u + m in float32.
template <int CPL>
__device__ __forceinline__ void load_kivi_k(const LayerView& lv, const uint8_t* kreg, const float* pend, long long pos,
                                            long long entered, int lane, float (&x)[CPL]) {
    const int D = lv.D;
    if (pos >= entered / 32 * 32) {
        const float* r = pend + (pos % 32) * D + lane * CPL;
#pragma unroll
        for (int j = 0; j < CPL; ++j) x[j] = r[j];
        return;
    }
    const RowFmt f = lv.fmt[0];
    const int t = (int)(pos % 32);
    const int off = 1 << (f.bits - 1);
    const int p0 = f.asym ? 4 : 2, p1 = p0 + 4 * f.w0;
    const uint32_t m0 = (1u << f.w0) - 1, m1 = (1u << f.w1) - 1;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        const uint8_t* blk = kreg + ((pos / 32) * D + lane * CPL + j) * (long long)lv.kbb;
        const float d = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(blk)));
        uint32_t u = (blk[p0 + (t * f.w0) / 8] >> ((t * f.w0) % 8)) & m0;
        if (f.w1) u |= ((blk[p1 + (t * f.w1) / 8] >> ((t * f.w1) % 8)) & m1) << f.w0;
        if (f.asym) {
            const float m = __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(blk + 2)));
            x[j] = __fadd_rn(__fmul_rn(d, (float)u), m);
        } else {
            x[j] = __fmul_rn(d, (float)((int)u - off));
        }
    }
}

template <int CPL>
__global__ void __launch_bounds__(32 * P1_WARPS)
attn_pass1(P1Args a) {
    const LayerView& lv = a.lv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int D = lv.D, G = lv.G, H = lv.H;
    const int h = blockIdx.y;
    const int br = blockIdx.z;                 // b * rows + r
    const int b = br / a.rows, r = br % a.rows;
    const int split = blockIdx.x;
    const long long limit = a.pos_base + r;    // last position this row may see

    const long long t0 = (long long)split * a.chunk;
    long long t1 = t0 + a.chunk;
    if (t1 > a.region_rows) t1 = a.region_rows;
    if (!a.ring && !a.idx && t1 > limit + 1) t1 = limit + 1;   // main rows: index == position
    const int* il = a.idx ? a.idx + ((long long)br * H + h) * a.n_idx : nullptr;

    const int kvarn = lv.kvarn && !a.ring;
    const float* sK = kvarn ? lv.scales + ((long long)(b * H + h) * 2 + 0) * D : nullptr;
    const float* sV = kvarn ? lv.scales + ((long long)(b * H + h) * 2 + 1) * D : nullptr;

    // q for the G heads of this kv head, this lane's channels, pre-scaled
    float qr[MAXG][CPL];
    const float* qb = a.q + ((long long)br * lv.G * H + (long long)h * G) * D;
#pragma unroll
    for (int g = 0; g < MAXG; ++g) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            const int c = lane * CPL + j;
            float v = (g < G) ? qb[(long long)g * D + c] * a.qscale : 0.f;
            if (kvarn) v *= sK[c];
            qr[g][j] = v;
        }
    }

    const RowFmt fk = a.ring ? lv.tail : lv.fmt[0];
    const RowFmt fv = a.ring ? lv.tail : lv.fmt[1];
    const uint8_t* kbase = a.ring ? lv.ring[0] + (long long)(b * H + h) * lv.ring_region
                                  : lv.main[0] + (long long)(b * H + h) * lv.main_region[0];
    const uint8_t* vbase = a.ring ? lv.ring[1] + (long long)(b * H + h) * lv.ring_region
                                  : lv.main[1] + (long long)(b * H + h) * lv.main_region[1];
    const long long ring_base = a.n - lv.W;    // ring slot s holds position ring_base + ((s - ring_base) mod W)

    float m[MAXG], l[MAXG], o[MAXG][CPL];
#pragma unroll
    for (int g = 0; g < MAXG; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) o[g][j] = 0.f;
    }

    for (long long t = t0 + warp; t < t1; t += P1_WARPS) {
        long long row = t;
        if (il) {
            // gather: list entry t names a position; this pass takes those of its region
            const long long p = il[t];
            const long long ring0 = lv.W ? a.n - lv.W : a.n;
            if (a.ring) {
                if (p < 0 || p < ring0 || p >= a.n) continue;
                row = p % lv.W;
            } else {
                if (p < 0 || p >= ring0) continue;
                row = p;
            }
        } else if (a.ring) {
            const long long W = lv.W;
            const long long pos = ring_base + ((t - ring_base) % W + W) % W;
            if (pos > limit) continue;
        }
        float kx[CPL], vx[CPL];
        if (lv.kivi && !a.ring)
            load_kivi_k<CPL>(lv, kbase, lv.pend + (long long)(b * H + h) * 32 * D, row,
                             lv.W ? a.n - (a.n < lv.W ? a.n : lv.W) : a.n, lane, kx);
        else
            load_row_values<CPL>(kbase + row * fk.stride, fk, lane, kx);
        load_row_values<CPL>(vbase + row * fv.stride, fv, lane, vx);
        float s[MAXG];
#pragma unroll
        for (int g = 0; g < MAXG; ++g) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < CPL; ++j) acc = fmaf(qr[g][j], kx[j], acc);
            s[g] = acc;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
#pragma unroll
            for (int g = 0; g < MAXG; ++g)
                if (g < G) s[g] += __shfl_xor_sync(0xffffffffu, s[g], off);
        }
#pragma unroll
        for (int g = 0; g < MAXG; ++g) {
            if (g >= G) break;
            if (s[g] > m[g]) {
                const float corr = exp2f(m[g] - s[g]);
                l[g] *= corr;
#pragma unroll
                for (int j = 0; j < CPL; ++j) o[g][j] *= corr;
                m[g] = s[g];
            }
            const float p = exp2f(s[g] - m[g]);
            l[g] += p;
#pragma unroll
            for (int j = 0; j < CPL; ++j) o[g][j] = fmaf(p, vx[j], o[g][j]);
        }
    }

    // combine the warps of this CTA
    __shared__ float sm_m[P1_WARPS][MAXG], sm_l[P1_WARPS][MAXG];
    extern __shared__ float sm_o[];            // [P1_WARPS][G][D]
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < MAXG; ++g) { sm_m[warp][g] = m[g]; sm_l[warp][g] = l[g]; }
    }
#pragma unroll
    for (int g = 0; g < MAXG; ++g) {
        if (g >= G) break;
#pragma unroll
        for (int j = 0; j < CPL; ++j) sm_o[((warp * G) + g) * D + lane * CPL + j] = o[g][j];
    }
    __syncthreads();

    float* part = a.ws + ((((long long)br * H + h) * a.n_split) + a.split_offset + split) * ((long long)G * (D + 2));
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int g = idx / D, c = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < P1_WARPS; ++w) M = fmaxf(M, sm_m[w][g]);
        float O = 0.f, L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < P1_WARPS; ++w) {
                const float e = exp2f(sm_m[w][g] - M);
                O = fmaf(sm_o[((w * G) + g) * D + c], e, O);
                L = fmaf(sm_l[w][g], e, L);
            }
        }
        if (sV) O *= sV[c];
        part[2 * G + idx] = O;
        if (c == 0) { part[g] = M; part[G + g] = L; }
    }
}

// Merge of the split partials. One CTA per (b, row, q head) and 32-channel slice; its
// 32 * MG threads are 32 channels x MG split groups. Group j folds splits j, j+MG, ... in
// order with an online rescale (one pass over m, l and o), then the MG groups are folded
// in a fixed order, so the result is bit-reproducible.
constexpr int MG = 16;
constexpr int MU = 4;   // partials per merge step

__global__ void __launch_bounds__(32 * MG) attn_merge(const float* __restrict__ ws, float* __restrict__ out, int G,
                                                  int H, int D, int n_split) {
    __shared__ float sm_m[MG][32], sm_l[MG][32], sm_o[MG][32];
    const int hq = blockIdx.x % (G * H);
    const long long br = blockIdx.x / (G * H);
    const int h = hq / G, g = hq % G;
    const long long stride = (long long)G * (D + 2);
    const float* base = ws + ((br * H + h) * n_split) * stride;
    const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
    asm volatile("griddepcontrol.wait;" ::: "memory");   // partials of the preceding pass(es)

    const int c = blockIdx.y * 32 + lane;
    const int cc = c < D ? c : D - 1;
    float M = -INFINITY, L = 0.f, O = 0.f;
    // MU partials per step: their loads are independent and in flight together; one rescale
    // of the running sums per step
    for (int s0 = grp; s0 < n_split; s0 += MG * MU) {
        float ms[MU], ls[MU], os[MU];
#pragma unroll
        for (int u = 0; u < MU; ++u) {
            const int s = s0 + u * MG;
            ms[u] = -INFINITY; ls[u] = 0.f; os[u] = 0.f;
            if (s < n_split) {
                const float* ps = base + (long long)s * stride;
                ms[u] = ps[g]; ls[u] = ps[G + g]; os[u] = ps[2 * G + (long long)g * D + cc];
            }
        }
        float mx = M;
#pragma unroll
        for (int u = 0; u < MU; ++u) mx = fmaxf(mx, ms[u]);
        if (mx == -INFINITY) continue;
        if (mx > M) {
            const float e = (M == -INFINITY) ? 0.f : exp2f(M - mx);
            L *= e;
            O *= e;
            M = mx;
        }
#pragma unroll
        for (int u = 0; u < MU; ++u) {
            if (ms[u] == -INFINITY) continue;
            const float w = exp2f(ms[u] - M);
            L = fmaf(ls[u], w, L);
            O = fmaf(os[u], w, O);
        }
    }
    sm_m[grp][lane] = M;
    sm_l[grp][lane] = L;
    sm_o[grp][lane] = O;
    __syncthreads();
    if (grp == 0 && c < D) {
        float Mt = -INFINITY;
        for (int j = 0; j < MG; ++j) Mt = fmaxf(Mt, sm_m[j][lane]);
        float Lt = 0.f, Ot = 0.f;
        for (int j = 0; j < MG; ++j) {
            const float mj = sm_m[j][lane];
            if (mj == -INFINITY) continue;
            const float w = exp2f(mj - Mt);
            Lt = fmaf(sm_l[j][lane], w, Lt);
            Ot = fmaf(sm_o[j][lane], w, Ot);
        }
        // no position at all (an index list without a valid entry): zero output
        out[(br * H * G + hq) * (long long)D + c] = Lt > 0.f ? Ot / Lt : 0.f;
    }
}

template <int CPL>
cudaError_t run_pass1(const P1Args& a, int n_region_split, int B, cudaStream_t st) {
    if (n_region_split == 0) return cudaSuccess;
    const dim3 grid(n_region_split, a.lv.H, B * a.rows);
    const size_t smem = (size_t)P1_WARPS * a.lv.G * a.lv.D * sizeof(float);
    attn_pass1<CPL><<<grid, 32 * P1_WARPS, smem, st>>>(a);
    return cudaGetLastError();
}

// One warp waits, with the pipelines' bounded wait, on an mbarrier that nothing arrives on;
// the wait runs out after limit_ns and the timeout is recorded like a pipeline's would be.
__global__ void wait_selftest(uint32_t* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mma::mbar_init(&bar, 1);
        mma::fence_mbar_init();
    }
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, mma::mbar_wait(&bar, 0, limit_ns, false)) != 0;
    if (!ok && threadIdx.x == 0) atomicOr(status, STATUS_WAIT_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_selftest(uint32_t* status, unsigned long long limit_ns, cudaStream_t st) {
    wait_selftest<<<1, 32, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

size_t partial_floats(int G, int D) { return (size_t)G * (D + 2); }

bool use_tensor_cores(int D) { return D == 128 || D == 256; }

int tc_ctas_per_sm(int head_dim) { return tc::min_ctas(head_dim / 32); }

SplitPlan plan_splits(long long n_main, long long n_ring, long long units, int num_sms, int tc_ctas) {
    SplitPlan p{};
    const bool tc = tc_ctas > 0;
    const long long target = (tc ? (long long)tc_ctas : 4LL) * num_sms;
    // rounded down: units * per_unit CTAs must not spill into a second wave
    long long per_unit = target / units;
    if (per_unit < 1) per_unit = 1;
    if (tc) {
        // every split of either region gets the same number of tiles, chosen so that both
        // regions' splits fit in about one wave (per_unit per unit, tc_ctas CTAs per SM): the ring
        // pass and the low-bit pass then run side by side and end together
        const long long tr = (n_ring + tc::TOK - 1) / tc::TOK, tm = (n_main + tc::TOK - 1) / tc::TOK;
        long long per = (tr + tm + per_unit - 1) / per_unit;
        if (per < 1) per = 1;
        // each region rounds its split count up: grow the tile count until both fit
        while ((tr + per - 1) / per + (tm + per - 1) / per > per_unit && per < tr + tm) ++per;
        p.ring_chunk = p.main_chunk = per * tc::TOK;
        p.n_ring_split = (int)((tr + per - 1) / per);
        p.n_main_split = (int)((tm + per - 1) / per);
        return p;
    }
    // CUDA-core path: about per_unit splits per region, low-bit splits of at least 64 rows
    const long long align = 16;
    long long rchunk = (n_ring + per_unit - 1) / per_unit;
    if (rchunk < align) rchunk = align;
    rchunk = (rchunk + align - 1) / align * align;
    long long chunk = (n_main + per_unit - 1) / per_unit;
    if (chunk < 4 * align) chunk = 4 * align;
    chunk = (chunk + align - 1) / align * align;
    p.ring_chunk = rchunk;
    p.main_chunk = chunk;
    p.n_ring_split = (int)((n_ring + rchunk - 1) / rchunk);
    p.n_main_split = (int)((n_main + chunk - 1) / chunk);
    return p;
}

cudaError_t launch_attention(const LayerView& lv, const float* q, float scale, float* out,
                             float* ws, long long n, int rows, const SplitPlan& plan,
                             cudaStream_t st, const int* idx, int n_idx) {
    P1Args a{};
    a.idx = idx;
    a.n_idx = n_idx;
    a.lv = lv;
    a.q = q;
    a.qscale = scale * LOG2E;
    a.ws = ws;
    a.n = n;
    a.pos_base = n - rows;
    a.rows = rows;
    a.n_split = plan.n_split();
    const long long n_ring = lv.W ? (n < lv.W ? n : (long long)lv.W) : 0;
    const long long n_main = n - n_ring;
    const int CPL = lv.D / 32;
    const bool tcp = use_tensor_cores(lv.D) && !lv.kivi;   // per-channel K: CUDA-core path
    int launched = 0;
    // the ring pass goes first: its few short splits take their SM slots before the
    // low-bit pass fills the rest, instead of waiting for low-bit splits to retire
    for (int ri = 0; ri < 2; ++ri) {
        const int region = 1 - ri;
        a.ring = region;
        a.chunk = region ? plan.ring_chunk : plan.main_chunk;
        a.region_rows = idx ? n_idx : (region ? n_ring : n_main);
        a.split_offset = region ? plan.n_main_split : 0;
        const int ns = region ? plan.n_ring_split : plan.n_main_split;
        if (ns == 0) continue;
        cudaError_t e;
        if (tcp) {
            tc::Args t{};
            const RowFmt& fk = region ? lv.tail : lv.fmt[0];
            const RowFmt& fv = region ? lv.tail : lv.fmt[1];
            t.kbase = region ? lv.ring[0] : lv.main[0];
            t.vbase = region ? lv.ring[1] : lv.main[1];
            t.kstride = fk.stride;
            t.vstride = fv.stride;
            t.q = q;
            t.qscale = a.qscale;
            t.scales = lv.kvarn ? lv.scales : nullptr;
            t.stats = lv.stats;
            t.status = lv.status;
            t.ws = ws;
            t.n = n;
            t.pos_base = a.pos_base;
            t.rows = rows;
            t.ring = region;
            t.W = lv.W;
            t.chunk = a.chunk;
            t.region_rows = a.region_rows;
            t.region_stride_k = region ? lv.ring_region : lv.main_region[0];
            t.region_stride_v = region ? lv.ring_region : lv.main_region[1];
            t.split_offset = a.split_offset;
            t.n_split = a.n_split;
            t.H = lv.H;
            t.G = lv.G;
            t.D = lv.D;
            t.idx = idx;
            t.n_idx = n_idx;
            t.ring_start = lv.W ? n - lv.W : n;
            t.dependent = launched ? 1 : 0;
            const dim3 grid(ns, lv.H, lv.B * rows);
            e = tc::launch_tc(fk.id, fv.id, t, grid, tc::smem_bytes(fk.stride, fv.stride, lv.D, tc::query_parts(fk.id)), st);
        } else {
            switch (CPL) {
                case 1: e = run_pass1<1>(a, ns, lv.B, st); break;
                case 2: e = run_pass1<2>(a, ns, lv.B, st); break;
                case 4: e = run_pass1<4>(a, ns, lv.B, st); break;
                case 8: e = run_pass1<8>(a, ns, lv.B, st); break;
                default: return cudaErrorInvalidValue;
            }
        }
        if (e != cudaSuccess) return e;
        ++launched;
    }
    // the merge is a programmatic dependent: it launches early and waits for the passes
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((long long)lv.B * rows * lv.H * lv.G), (unsigned)((lv.D + 31) / 32));
    cfg.blockDim = dim3(32 * MG);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_merge, (const float*)ws, out, lv.G, lv.H, lv.D, a.n_split);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace kvq
