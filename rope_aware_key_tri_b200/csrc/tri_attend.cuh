// tri_attend.cuh -- decode attention over a pruned cache, for sm_100a.
//
// The consumer of the compacted cache: for every query head h of a unit (sequence s, layer l,
// KV head g), the standard scaled dot-product attention over the unit's cached rows,
//   out_h = sum_i softmax_i(q_h . k_i / sqrt(d)) v_i,
// as the page "TriAttention 深度解析：MIT韩松团队如何用三角函数让单卡4090跑出百万Token上下文"
// writes it out in its section 二 ("TriAttention的核心发现"). The query is post-RoPE (rotated at
// its own position) like the stored keys, so every logit already depends on the distance only
// and the kept keys' scattered positions need nothing else.
//
// Work: one CTA per (unit, chunk of keys). The unit's rows are split into `cpu` chunks when
// there are too few units to fill the GPU; each CTA streams its chunk's K and V rows once from
// HBM (TMA bulk copies into per-warp buffers, 16 rows per stage, evict-first) and keeps, per
// query head, the running maximum m, the running sum l and the weighted sum of values acc
// (online softmax, log2 domain, fp32). A key is split over LPK = d/8 lanes of a warp, each lane
// holding 8 dims of the G query rows; the lanes' partial dot products are summed with
// shuffles. A chunk's (m, l, acc) go to a partial buffer that the combine kernel merges; a
// unit held by one chunk is normalised and written directly.
//
// Bound: HBM (2 * 2d bytes per kept key against 4 G d flops: 4 flop/B at G = 4, 8 at G = 8,
// below the CUDA-core ridge), so no tensor cores.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tri_kernel.cuh"

namespace tri {

constexpr int kAttWarps = 4;
constexpr int kAttThreads = kAttWarps * 32;
constexpr int kAttStageRows = 16;

struct AttArgs {
    const uint16_t *K;           // bf16 bits, the cache layout of tri_kv
    const uint16_t *V;
    const uint16_t *q;           // [n_layers][batch][Hq][D] bf16 post-RoPE queries
    float *out;                  // [n_layers][batch][Hq][D]
    float *part;                 // [n_units][cpu][G][D + 2] chunk partials: acc[D], then m, l
    const int32_t *lens;
    const int32_t *block_table;
    const int32_t *seq_bad;      // validation verdicts (a refused sequence is not written)
    int batch, n_kv, cap_u;
    int paged, page_size, max_pages, n_pages;
    int n_units;
    int cpu;                     // chunks per unit
    int nslot;                   // TMA stages per warp
    float qscale;                // log2(e) / sqrt(D): logits in the log2 domain
    unsigned long long *status;
    int wait_tries;
    long long unit_base;
};

template <int D, int G>
struct AttGeo {
    // dims per lane: 8 keeps the query slices and accumulators small enough (167 registers at
    // G = 4) for three CTAs per SM, which measured 5 % faster than 16 dims at two CTAs
    static constexpr int DPL = 8;
    static constexpr int LPK = D / DPL;          // lanes per key
    static constexpr int KPP = 32 / LPK;         // keys per warp pass
    static constexpr int PASSES = kAttStageRows / KPP;
    static constexpr int SB = PASSES < 32 / G ? PASSES : 32 / G;  // keys per rescale (<= 32 logits)
    static_assert(LPK >= 2 && 32 % LPK == 0 && KPP <= kAttStageRows, "lane geometry");
};

__host__ __device__ inline unsigned att_stage_bytes(int D) { return 2u * kAttStageRows * (unsigned)D * 2u; }
__host__ __device__ inline unsigned att_smem_bytes(int D, int G, int nslot) {
    // per-warp stages (K then V), the per-warp barriers, and the cross-warp combine area
    return (unsigned)kAttWarps * nslot * att_stage_bytes(D) + (unsigned)kAttWarps * nslot * 8u +
           (unsigned)kAttWarps * G * (D + 2) * 4u;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Rows [k0, k1) of unit (lr, s, g) -> the chunk's (m, l, acc) per head; written as a partial,
// or normalised into out when the unit is one chunk.
template <int D, int G>
__global__ void __launch_bounds__(kAttThreads) tri_attend_kernel(const AttArgs a) {
    using GE = AttGeo<D, G>;
    constexpr int DPL = GE::DPL, LPK = GE::LPK, KPP = GE::KPP, PASSES = GE::PASSES, SB = GE::SB;
    constexpr unsigned FULL = 0xffffffffu;
    const float NEG_INF = __int_as_float(0xff800000);
    extern __shared__ __align__(128) unsigned char att_smem[];
    const int nslot = a.nslot;
    const unsigned stage_bytes = att_stage_bytes(D);
    uint64_t *bars = reinterpret_cast<uint64_t *>(att_smem + (size_t)kAttWarps * nslot * stage_bytes);
    float *xw = reinterpret_cast<float *>(att_smem + (size_t)kAttWarps * nslot * stage_bytes +
                                          (size_t)kAttWarps * nslot * 8u);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int unit = blockIdx.x / a.cpu, chunk = blockIdx.x % a.cpu;
    const int g = unit % a.n_kv;
    const int s = (unit / a.n_kv) % a.batch;
    const int lr = unit / (a.n_kv * a.batch);
    const int Hq = a.n_kv * G;
    // a programmatic dependent of the validation kernel: its verdicts are read after this
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int N = __ldg(a.lens + s);
    if (__ldg(a.seq_bad + s) != 0 || N < 0 || N > a.cap_u) return;  // uniform: nothing is written
    const int per = ((N + a.cpu - 1) / a.cpu + kAttStageRows - 1) / kAttStageRows * kAttStageRows;
    const int k0 = min(N, chunk * per), k1 = min(N, k0 + per);
    const int n_local = k1 - k0;
    const int nst = (n_local + kAttStageRows - 1) / kAttStageRows;
    const int my_stages = warp < nst ? (nst - warp + kAttWarps - 1) / kAttWarps : 0;

    const int sub = lane % LPK, kw = lane / LPK;
    const long long qrow = (((long long)lr * a.batch + s) * Hq + (long long)g * G) * D;

    if (lane == 0) {
        for (int k = 0; k < nslot; ++k) mbar_init(bars + warp * nslot + k, 1);
        mbar_init_fence();
    }
    __syncwarp();
    const uint64_t pol = policy_evict_first();
    unsigned char *ring = att_smem + (size_t)warp * nslot * stage_bytes;
    auto issue = [&](int st, int slot) {
        const int r0 = st * kAttStageRows;
        const int nrows = min(kAttStageRows, n_local - r0);
        const int i0 = k0 + r0;
        long long row;
        if (!a.paged) {
            row = (((long long)lr * a.batch + s) * a.n_kv + g) * (long long)a.cap_u + i0;
        } else {
            const int pg = __ldg(a.block_table + (long long)s * a.max_pages + i0 / a.page_size);
            row = (((long long)lr * a.n_pages + pg) * a.n_kv + g) * (long long)a.page_size + (i0 % a.page_size);
        }
        uint64_t *bar = bars + warp * nslot + slot;
        unsigned char *dst = ring + (size_t)slot * stage_bytes;
        const unsigned bytes = (unsigned)nrows * D * 2u;
        fence_proxy_async_smem();
        mbar_expect_tx(bar, 2u * bytes);
        tma_load_1d(dst, a.K + row * D, bytes, bar, pol);
        tma_load_1d(dst + stage_bytes / 2, a.V + row * D, bytes, bar, pol);
    };
    const int pre = min(nslot, my_stages);
    if (lane == 0)
        for (int k = 0; k < pre; ++k) issue(warp + k * kAttWarps, k);

    // the lane's slice of the G query rows, scaled into the log2 domain
    // (pairs of dims: element 2j and 2j + 1 of the lane's slice)
    float2 qf[G][DPL / 2];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const uint4 *qp = reinterpret_cast<const uint4 *>(a.q + qrow + (long long)h * D + sub * DPL);
#pragma unroll
        for (int c = 0; c < DPL / 8; ++c) {
            const uint4 x = __ldg(qp + c);
            const unsigned w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) qf[h][4 * c + e] = make_float2(bf16lo(w[e]) * a.qscale, bf16hi(w[e]) * a.qscale);
        }
    }

    float m[G], l[G];
    float2 acc[G][DPL / 2];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = NEG_INF;
        l[h] = 0.f;
#pragma unroll
        for (int i = 0; i < DPL / 2; ++i) acc[h][i] = make_float2(0.f, 0.f);
    }

    bool ok = true;
    int slot = 0;
    unsigned phase = 0;
    for (int k = 0; k < my_stages; ++k) {
        const int st = warp + k * kAttWarps;
        if (!__all_sync(FULL, mbar_wait_bounded(bars + warp * nslot + slot, phase, a.wait_tries))) {
            // let the copies still in flight for this warp land (bounded), then give up
            int sl = slot;
            unsigned ph = phase;
            for (int j = k + 1; j < min(my_stages, k + nslot); ++j) {
                if (++sl == nslot) { sl = 0; ph ^= 1u; }
                (void)mbar_wait_bounded(bars + warp * nslot + sl, ph, a.wait_tries);
            }
            ok = false;
            break;
        }
        const uint16_t *Ks = reinterpret_cast<const uint16_t *>(ring + (size_t)slot * stage_bytes);
        const uint16_t *Vs = Ks + kAttStageRows * D;
        const int valid = n_local - st * kAttStageRows;  // rows of this stage
        // the lane group's keys of the stage in sub-blocks of SB: logits, one rescale, then the
        // weighted values
#pragma unroll
        for (int p0 = 0; p0 < PASSES; p0 += SB) {
            float sv[SB][G];
#pragma unroll
            for (int pp = 0; pp < SB; ++pp) {
                const int r = (p0 + pp) * KPP + kw;
                const uint16_t *kr = Ks + r * D + sub * DPL;
                float2 dot[G];
#pragma unroll
                for (int h = 0; h < G; ++h) dot[h] = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < DPL / 8; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(kr + 8 * c);
                    const unsigned w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 k2 = make_float2(bf16lo(w[e]), bf16hi(w[e]));
#pragma unroll
                        for (int h = 0; h < G; ++h) dot[h] = __ffma2_rn(qf[h][4 * c + e], k2, dot[h]);
                    }
                }
                float dsum[G];
#pragma unroll
                for (int h = 0; h < G; ++h) dsum[h] = dot[h].x + dot[h].y;
#pragma unroll
                for (int o = LPK / 2; o >= 1; o >>= 1)
#pragma unroll
                    for (int h = 0; h < G; ++h) dsum[h] += __shfl_xor_sync(FULL, dsum[h], o);
#pragma unroll
                for (int h = 0; h < G; ++h) sv[pp][h] = r < valid ? dsum[h] : NEG_INF;
            }
            // the running maxima only move when a logit of this sub-block exceeds them, which
            // after the first few sub-blocks is rare: the warp rescales only when some lane's did
            float mnew[G];
            bool grew = false;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float mb = sv[0][h];
#pragma unroll
                for (int pp = 1; pp < SB; ++pp) mb = fmaxf(mb, sv[pp][h]);
                mnew[h] = fmaxf(m[h], mb);
                grew |= mnew[h] > m[h];
            }
            if (__any_sync(FULL, grew)) {
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    if (mnew[h] != NEG_INF) {
                        const float corr = ex2_approx(m[h] - mnew[h]);  // 1 if unchanged, 0 from -inf
                        l[h] *= corr;
                        const float2 c2 = make_float2(corr, corr);
#pragma unroll
                        for (int i = 0; i < DPL / 2; ++i) acc[h][i] = __fmul2_rn(acc[h][i], c2);
                        m[h] = mnew[h];
                    }
                }
            }
#pragma unroll
            for (int pp = 0; pp < SB; ++pp) {
                const int r = (p0 + pp) * KPP + kw;
                const bool in = r < valid;
                float2 pr[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float pv = in ? ex2_approx(sv[pp][h] - m[h]) : 0.f;
                    l[h] += pv;
                    pr[h] = make_float2(pv, pv);
                }
                const uint16_t *vr = Vs + r * D + sub * DPL;
#pragma unroll
                for (int c = 0; c < DPL / 8; ++c) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(vr + 8 * c);
                    const unsigned w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // rows past the stage's end hold stale bits (maybe NaN): zero them
                        const float2 v2 = in ? make_float2(bf16lo(w[e]), bf16hi(w[e])) : make_float2(0.f, 0.f);
#pragma unroll
                        for (int h = 0; h < G; ++h) acc[h][4 * c + e] = __ffma2_rn(pr[h], v2, acc[h][4 * c + e]);
                    }
                }
            }
        }
        __syncwarp();
        if (k + nslot < my_stages && lane == 0) issue(st + nslot * kAttWarps, slot);
        if (++slot == nslot) { slot = 0; phase ^= 1u; }
    }
    if (__syncthreads_or(!ok)) {
        if (tid == 0) record_status(a.status, kDevTimeout, a.unit_base + unit);
        return;  // every copy this CTA issued has landed or been waited for (bounded)
    }

    // merge the warp's lane groups (keys kw), then the warps, in a fixed order
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float mo = __shfl_xor_sync(FULL, m[h], o);
            const float lo = __shfl_xor_sync(FULL, l[h], o);
            const float mn = fmaxf(m[h], mo);
            const float ca = mn == NEG_INF ? 0.f : ex2_approx(m[h] - mn);
            const float cb = mn == NEG_INF ? 0.f : ex2_approx(mo - mn);
            l[h] = l[h] * ca + lo * cb;
#pragma unroll
            for (int i = 0; i < DPL / 2; ++i) {
                const float ax = __shfl_xor_sync(FULL, acc[h][i].x, o);
                const float ay = __shfl_xor_sync(FULL, acc[h][i].y, o);
                acc[h][i] = make_float2(acc[h][i].x * ca + ax * cb, acc[h][i].y * ca + ay * cb);
            }
            m[h] = mn;
        }
    }
    // per warp: xw[warp][h] = acc[D], m, l
    if (kw == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float *row = xw + ((size_t)warp * G + h) * (D + 2);
#pragma unroll
            for (int i = 0; i < DPL / 2; ++i) {
                row[sub * DPL + 2 * i] = acc[h][i].x;
                row[sub * DPL + 2 * i + 1] = acc[h][i].y;
            }
            if (sub == 0) {
                row[D] = m[h];
                row[D + 1] = l[h];
            }
        }
    }
    __syncthreads();
    const bool direct = a.cpu == 1;
    for (int idx = tid; idx < G * (D + 2); idx += kAttThreads) {
        const int h = idx / (D + 2), i = idx % (D + 2);
        float M = NEG_INF;
        for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, xw[((size_t)w * G + h) * (D + 2) + D]);
        float L = 0.f, A = 0.f;
        for (int w = 0; w < kAttWarps; ++w) {
            const float *row = xw + ((size_t)w * G + h) * (D + 2);
            const float c = M == NEG_INF ? 0.f : ex2_approx(row[D] - M);
            L += row[D + 1] * c;
            if (i < D) A += row[i] * c;
        }
        if (direct) {
            if (i < D) a.out[qrow + (long long)h * D + i] = L > 0.f ? A / L : 0.f;
        } else {
            float *pp = a.part + (((long long)unit * a.cpu + chunk) * G + h) * (D + 2);
            pp[i] = i < D ? A : (i == D ? M : L);
        }
    }
}

// Merge the chunks of every unit: out_h = sum_c acc_c 2^(m_c - M) / sum_c l_c 2^(m_c - M).
template <int D, int G>
__global__ void __launch_bounds__(256) tri_attend_combine_kernel(const AttArgs a) {
    const float NEG_INF = __int_as_float(0xff800000);
    const int unit = blockIdx.x;
    const int g = unit % a.n_kv;
    const int s = (unit / a.n_kv) % a.batch;
    const int lr = unit / (a.n_kv * a.batch);
    // a programmatic dependent of the attention kernel: the partials are read after this
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int N = __ldg(a.lens + s);
    if (__ldg(a.seq_bad + s) != 0 || N < 0 || N > a.cap_u) return;
    const long long qrow = (((long long)lr * a.batch + s) * (a.n_kv * G) + (long long)g * G) * D;
    const int per = ((N + a.cpu - 1) / a.cpu + kAttStageRows - 1) / kAttStageRows * kAttStageRows;
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, i = idx % D;
        float M = NEG_INF;
        for (int c = 0; c < a.cpu; ++c) {
            if (c * per >= N) break;  // chunks past the length were not run
            M = fmaxf(M, a.part[(((long long)unit * a.cpu + c) * G + h) * (D + 2) + D]);
        }
        float L = 0.f, A = 0.f;
        for (int c = 0; c < a.cpu; ++c) {
            if (c * per >= N) break;
            const float *pp = a.part + (((long long)unit * a.cpu + c) * G + h) * (D + 2);
            const float w = M == NEG_INF ? 0.f : ex2_approx(pp[D] - M);
            L += pp[D + 1] * w;
            A += pp[i] * w;
        }
        a.out[qrow + (long long)h * D + i] = L > 0.f ? A / L : 0.f;
    }
}

}  // namespace tri
