// tri_calib.cuh -- calibration statistics from pre-RoPE query samples, for sm_100a.
//
// Pages cited (titles; sections as headed on each page):
//   [Deep-dive]  "TriAttention深度解析：用三角函数革命性压缩KV Cache，让长推理从「显存地狱」中脱困"
//   [Stage]      "旋转舞台上的追光者——TriAttention如何用三角函数破解长文本推理的内存困局"
//
// The offline calibration of [Deep-dive] §3.4 runs a small batch (about 10K tokens) through
// the model and keeps, per attention head, the query centre, the mean norm and the
// concentration R. Per band f of query head h of layer l, over the T calibration tokens:
//   E[q_f]  = mean_t q_f(t)                  (complex; [Stage] §TriAttention：把理论变成算法 item 1)
//   E|q_f|  = mean_t |q_f(t)|                ([Stage] item 2)
//   R_f     = |E[q_f]| / E|q_f|              ([Stage] §破局之道, taken per band; 0 for a band
//                                            whose samples are all zero)
//
// The pass is one stream over Q (HBM-bound): a CTA takes a fixed chunk of tokens of one
// layer and 128 threads; each thread owns 4 bands of one head (16 bytes per token: two 8-byte
// pieces in the half layout, where a band's two dims sit d/2 apart, one 16-byte piece in the
// interleaved layout), sums re, im and |q_f| (from the exact bf16 components: one fp32
// rounding of re^2 + im^2, a correctly rounded fp32 square root) over the chunk, and writes its
// chunk's sums; 8 tokens are loaded before any is used, added in fp32 (re and im as one packed
// pair), and each 8-token partial is added to fp64 chunk sums. A partial of 8 values is off by
// at most 7 * 2^-24 of the sum of their magnitudes (4.2e-7); the fp64 sums add nothing
// measurable. A second launch adds the chunks in order, so the result does not depend on the
// GPU, and forms the means and R.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tri {

constexpr int kCalThreads = 128;
constexpr int kCalMinBlocks = 6;  // CTAs per SM (24 warps hide the fp64 dependency latency)
constexpr int kCalBands = 4;      // bands per thread
constexpr int kCalChunk = 256;    // tokens per partial sum (fixed: the summation order is part of the result)
constexpr int kCalUnroll = 8;     // tokens in flight per thread

__device__ __forceinline__ float cal_lo(unsigned w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float cal_hi(unsigned w) { return __uint_as_float(w & 0xffff0000u); }

// part: [n_chunks][L][Hq][F][3] fp64 (sum re, sum im, sum |q_f|)
// A thread owns kCalBands bands of one head: its re and im dims are two 8-byte pieces in the
// half layout (d/2 dims apart) and one 16-byte piece in the interleaved layout.
template <int D, int LAYOUT>
__global__ void __launch_bounds__(kCalThreads, kCalMinBlocks) tri_calib_partial_kernel(const uint16_t *__restrict__ Q,
                                                                                    int L, int T, int Hq,
                                                                                    double *__restrict__ part) {
    constexpr int F = D / 2;
    constexpr int NB = kCalBands;
    constexpr int SLOTS = F / NB;  // column slots per head
    const int col = blockIdx.z * kCalThreads + threadIdx.x;
    if (col >= Hq * SLOTS) return;  // no barrier in this kernel
    const int chunk = blockIdx.x, l = blockIdx.y;
    const int h = col / SLOTS, slot = col % SLOTS;
    const int t0 = chunk * kCalChunk;
    const int t1 = min(T, t0 + kCalChunk);
    // element offset of the thread's re piece (half) or band piece (interleaved) in a token row
    const int off = LAYOUT == 0 ? h * D + slot * NB : h * D + slot * 2 * NB;
    const size_t row = (size_t)Hq * D;
    const uint16_t *base = Q + (size_t)l * T * row;

    double sr[NB], si[NB], sm[NB];
#pragma unroll
    for (int k = 0; k < NB; ++k) sr[k] = si[k] = sm[k] = 0.0;
    float2 pri[NB];  // fp32 partials of the current batch: (re, im) and |q_f|
    float pm[NB];
    // one token's pieces (four 32-bit words: 4 bands) into the batch partials
    auto add = [&](uint4 w) {
        const unsigned wv[4] = {w.x, w.y, w.z, w.w};
        float re[NB], im[NB];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            if (LAYOUT == 0) {
                // words 0-1: re of bands 0..3; words 2-3: their im
                re[2 * k] = cal_lo(wv[k]);
                re[2 * k + 1] = cal_hi(wv[k]);
                im[2 * k] = cal_lo(wv[2 + k]);
                im[2 * k + 1] = cal_hi(wv[2 + k]);
            } else {
                // each word is one band (re, im)
                re[2 * k] = cal_lo(wv[2 * k]);
                im[2 * k] = cal_hi(wv[2 * k]);
                re[2 * k + 1] = cal_lo(wv[2 * k + 1]);
                im[2 * k + 1] = cal_hi(wv[2 * k + 1]);
            }
        }
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            pri[k] = __fadd2_rn(pri[k], make_float2(re[k], im[k]));
            pm[k] += __fsqrt_rn(fmaf(re[k], re[k], im[k] * im[k]));
        }
    };
    auto clear = [&]() {
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            pri[k] = make_float2(0.f, 0.f);
            pm[k] = 0.f;
        }
    };
    auto flush = [&]() {
#pragma unroll
        for (int k = 0; k < NB; ++k) {
            sr[k] += (double)pri[k].x;
            si[k] += (double)pri[k].y;
            sm[k] += (double)pm[k];
        }
    };
    auto load = [&](int t) {
        const uint16_t *r = base + (size_t)t * row + off;
        if (LAYOUT == 0) {
            const uint2 a = __ldg(reinterpret_cast<const uint2 *>(r));
            const uint2 b = __ldg(reinterpret_cast<const uint2 *>(r + F));
            return make_uint4(a.x, a.y, b.x, b.y);
        }
        return __ldg(reinterpret_cast<const uint4 *>(r));
    };
    int t = t0;
    // whole batches: every load of the batch in flight before the first is used
    for (; t + kCalUnroll <= t1; t += kCalUnroll) {
        uint4 v[kCalUnroll];
#pragma unroll
        for (int u = 0; u < kCalUnroll; ++u) v[u] = load(t + u);
        clear();
#pragma unroll
        for (int u = 0; u < kCalUnroll; ++u) add(v[u]);
        flush();
    }
    // the chunk's ragged tail (the last chunk of a layer only): fewer than 8 tokens, one partial
    clear();
    for (; t < t1; ++t) add(load(t));
    flush();
    double *p = part + ((((size_t)chunk * L + l) * Hq + h) * F + (size_t)slot * NB) * 3;
#pragma unroll
    for (int k = 0; k < NB; ++k) {
        p[3 * k] = sr[k];
        p[3 * k + 1] = si[k];
        p[3 * k + 2] = sm[k];
    }
}

// One thread per (layer, head, band): chunk sums added in chunk order, then the means.
template <int D, int LAYOUT>
__global__ void __launch_bounds__(kCalThreads) tri_calib_final_kernel(const double *__restrict__ part, int n_chunks,
                                                                      int L, int T, int Hq, float *q_mean,
                                                                      float *q_norm_mean, float *R) {
    constexpr int F = D / 2;
    const long long i = (long long)blockIdx.x * kCalThreads + threadIdx.x;
    const long long nb = (long long)L * Hq * F;
    if (i >= nb) return;
    const int f = (int)(i % F);
    const long long lh = i / F;  // l * Hq + h
    double sr = 0.0, si = 0.0, sm = 0.0;
    for (int c = 0; c < n_chunks; ++c) {
        const double *p = part + ((size_t)c * nb + (size_t)i) * 3;
        sr += p[0];
        si += p[1];
        sm += p[2];
    }
    const double mr = sr / (double)T, mi = si / (double)T, mm = sm / (double)T;
    const int dre = LAYOUT == 0 ? f : 2 * f;
    const int dim = LAYOUT == 0 ? f + F : 2 * f + 1;
    q_mean[lh * D + dre] = (float)mr;
    q_mean[lh * D + dim] = (float)mi;
    q_norm_mean[i] = (float)mm;
    R[i] = mm > 0.0 ? (float)(sqrt(mr * mr + mi * mi) / mm) : 0.0f;
}

}  // namespace tri
