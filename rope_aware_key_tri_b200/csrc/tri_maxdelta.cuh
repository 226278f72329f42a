// tri_maxdelta.cuh -- scoring with the future offsets combined by the maximum, for sm_100a.
//
// Pages cited (titles; sections as headed on each page):
//   [Deep-dive]  "TriAttention深度解析：用三角函数革命性压缩KV Cache，让长推理从「显存地狱」中脱困"
//   [Stage]      "旋转舞台上的追光者——TriAttention如何用三角函数破解长文本推理的内存困局"
//   [10100]      the 10100.com article 127765992 on TriAttention
//
// [Deep-dive] §3.3 scores a key at every future offset delta of the geometric set and keeps
// the largest value (its §4.2 scoring code then adds the norm score). The maximum does not
// fold into one coefficient per band the way the mean does, so every key needs one dot
// product per (head, offset):
//   trig_{h,delta}(i) = sum_f Re(C_{h,delta,f} conj(k~_f(i))),
//   C_{h,delta,f}     = qbar_{h,f} e^{i omega_f (t + delta)}            (post-RoPE key k~)
//   s_h(i)            = max_delta trig_{h,delta}(i) + sum_f w_{h,f} |k~_f(i)|,  w = (1 - R) E|q|
// ([Stage] §TriAttention：把理论变成算法 items 1-2; the (1 - R) weight of [10100] §TriAttention方法).
// Per unit (sequence, layer, KV head) this is the product of the N x d key matrix with a
// d x (G |D|) coefficient matrix: a dense contraction, run on the tcgen05 tensor cores.
//
//   operands  A = 128 keys x d (bf16, straight from the cache by 2-D TMA with the 128-byte
//             swizzle), B = the unit's coefficient image: G |D| rows (padded to NCOL, a
//             multiple of 16) x d, in the same swizzled K-major layout, as a bf16 pair
//             hi + lo with hi = bf16(C), lo = bf16(C - hi), so that the product carries
//             about 16 significant bits of C while the key stays exact.
//   MMA       per 128-key tile: d/16 k-steps, each an M=128, N=NCOL, K=16 MMA for hi and one
//             for lo, both accumulating into the same fp32 TMEM accumulator.
//   epilogue  warpgroups of 4 warps take the tiles in turn, one TMEM lane (key) per
//             thread: the max over each head's columns (a head owns NOFF consecutive columns,
//             NOFF a compile-time count, the last offset repeated when the set is smaller,
//             so the max unrolls into three-input max instructions), plus the norm score from
//             the key row still in shared memory (packed fp32x2 FMAs); the scores go to a
//             [unit][slot][G] fp32 buffer that the fused kernel's z-score, select and
//             compaction read instead of scoring the keys themselves.
//
// One CTA per SM, warp-specialised: warp 0 issues the TMA loads, warp 1 owns the TMEM
// allocation and issues the MMAs, the other warps (three warpgroups, or two where the TMEM
// holds only two accumulators) run the epilogue. Key tiles stream through a ring of NST
// stages; the accumulators live in TMEM (tile k in buffer k mod NACC, its epilogue in
// warpgroup k mod NE); the coefficient image is double-buffered in shared memory and reloaded
// only when the CTA's tile range enters a new unit.
//
// The same kernel scores the mean over the offsets on the tensor cores (NOFF = 1): the
// coefficient of a head is then qbar A_f e^{i omega_f t}, the offset average folded in. Every wait is bounded; a wait that runs out records a device status, marks every unit
// of the CTA's tile range so that the fused kernel leaves them untouched, and ends the CTA's
// work.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tri_kernel.cuh"

namespace tri {

// Epilogue warpgroups (taking the tiles in turn): three where the TMEM holds three accumulators,
// else two. Threads per CTA: warp 0 issues the TMA loads, warp 1 the MMAs, then the epilogue.
__host__ __device__ constexpr int mx_epi_groups(int acc_cols) { return 512 / acc_cols >= 3 ? 3 : 2; }
__host__ __device__ constexpr int mx_threads_of(int acc_cols) { return 64 + 128 * mx_epi_groups(acc_cols); }
constexpr int kMxTile = 128;       // keys per tile (the MMA's M)
constexpr int kMxMaxStages = 6;
constexpr int kMxMaxAcc = 6;       // accumulator buffers the barrier block has room for
constexpr unsigned kMxChunkBytes = kMxTile * 128u;  // one 64-dim chunk of a tile: 128 rows x 128 B

// Columns per head: the offset count padded to one of three compile-time counts (the padding
// repeats the last offset, which leaves the maximum unchanged).
__host__ __device__ constexpr int mx_noff_pad(int n_off) { return n_off <= 1 ? 1 : n_off <= 17 ? 17 : 32; }
// Columns of the coefficient matrix: G NOFF rounded up to a multiple of 16 (M = 128 needs
// N % 16 == 0, 16 <= N <= 256).
__host__ __device__ constexpr int mx_ncol(int G, int noff) { return (G * noff + 15) / 16 * 16; }
// TMEM columns per accumulator buffer (a power of two, at least 32).
__host__ __device__ constexpr int mx_acc_cols(int ncol) {
    return ncol <= 32 ? 32 : ncol <= 64 ? 64 : ncol <= 128 ? 128 : 256;
}
// Accumulator buffers: one per epilogue warpgroup (so that one warpgroup owns every tile of a
// buffer), two per warpgroup where the 512 TMEM columns allow it.
__host__ __device__ constexpr int mx_nacc(int acc_cols) {
    return 512 / acc_cols >= 2 * mx_epi_groups(acc_cols) ? 2 * mx_epi_groups(acc_cols) : mx_epi_groups(acc_cols);
}
// Threads of the scoring kernel for head_dim-independent geometry (group, columns per head).
__host__ __device__ constexpr int mx_threads(int G, int noff) {
    return mx_threads_of(mx_acc_cols(noff == 1 ? 2 * mx_ncol(G, noff) : mx_ncol(G, noff)));
}
// Bytes of one half (hi or lo) of a coefficient image: d/64 chunks of NCOL rows x 128 B.
__host__ __device__ constexpr unsigned mx_half_bytes(int D, int ncol) { return (unsigned)(D / 64) * ncol * 128u; }
// Whole image: hi, lo, then the norm weights [G][F] fp32; a multiple of 1024 bytes.
__host__ __device__ inline unsigned mx_image_bytes(int D, int G, int ncol) {
    return align_up(2u * mx_half_bytes(D, ncol) + (unsigned)G * (D / 2) * 4u, 1024u);
}

struct MxArgs {
    const int32_t *lens;
    const int32_t *block_table;
    const int32_t *t;
    int batch, n_kv, cap_u;
    int paged, page_size, max_pages, n_pages;
    int layer_begin, n_layers;
    int min_len;                 // units with N <= min_len need no scores (prune: the budget)
    int n_off;                   // offsets per head
    int noffp;                   // columns per head (n_off padded)
    int ncol;                    // MMA N
    int nst;                     // key-tile stages
    int piece_rows;              // rows per TMA box (divides 128 and the page size)
    const double2 *qbar;         // [L][Hq][F] pre-RoPE query centres (complex)
    const double *omega;         // [F]
    const int64_t *offsets;      // [n_off]
    const float *w;              // [L][Hq][F] (1 - R) E|q|
    double2 *phase;              // [batch][n_off][F] e^{i omega_f (t_s + delta_j)}
    unsigned char *image;        // [n_units][image bytes]
    int32_t *tile_prefix;        // [batch + 1] tiles before sequence s in one layer (x n_kv)
    float *pre;                  // [n_units][cap_u][G] scores out
    int32_t *unit_fail;          // [n_units]
    unsigned long long *status;
    long long unit_base;         // added to the unit index in device status reports
    const int32_t *seq_bad;      // [batch] sequences refused by the validation kernel (no tiles)
    int wait_tries;              // tries (about 1 ms each) of every bounded wait
    long long inject_unit;       // test hook: the unit whose first key tile is withheld (-1: none)
    unsigned *unit_next;         // the fused kernel's unit counter, zeroed here for the launch after
};

// ---------------------------------------------------------------------------------
// Small PTX wrappers for TMA tiles, TMEM and the MMA.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), descriptor version 1.
__device__ __forceinline__ uint64_t mx_desc(const void *p) {
    const uint64_t a = (uint64_t)((smem_u32(p) >> 4) & 0x3FFFu);
    return a | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128, N = ncol.
__device__ __forceinline__ uint32_t mx_idesc(int ncol) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((unsigned)(ncol >> 3) << 17) | ((unsigned)(kMxTile >> 4) << 24);
}

__device__ __forceinline__ void mx_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mx_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 16 accumulator columns of this warp's 32 TMEM lanes, without waiting: the registers are valid
// after tmem_wait_ld (which takes them as operands, so no use can move above the wait).
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// 8 accumulator columns, without waiting (valid after tmem_wait_ld8 on the same registers).
__device__ __forceinline__ void tmem_ld8_issue(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld8(uint32_t (&a)[8], uint32_t (&b)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
                   "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]), "+r"(b[7])
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}

// Orders later uses of r after a tcgen05.wait::ld issued just before (no instruction).
__device__ __forceinline__ void tmem_after_wait(uint32_t (&r)[16]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// ---------------------------------------------------------------------------------
// Walk over the score tiles. Tiles are numbered layer by layer, sequence by sequence, KV
// head by KV head, 128 keys each; a CTA owns a contiguous range, so it stays on one unit for
// many tiles. Every role of the CTA walks the same range with its own copy.
// ---------------------------------------------------------------------------------
struct MxWalk {
    int lr, s, g, tile, tps, N;
    __device__ __forceinline__ static int tiles_of(const MxArgs &a, int s, int n) {
        return (n > a.min_len && n <= a.cap_u && __ldg(a.seq_bad + s) == 0) ? (n + kMxTile - 1) / kMxTile : 0;
    }
    __device__ __forceinline__ void start(const MxArgs &a, long long T, int per_layer) {
        lr = (int)(T / per_layer);
        const int x = (int)(T - (long long)lr * per_layer);
        int lo = 0, hi = a.batch;  // largest s with tile_prefix[s] <= x
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(a.tile_prefix + mid) <= x) lo = mid; else hi = mid;
        }
        s = lo;
        N = __ldg(a.lens + s);
        tps = tiles_of(a, s, N);
        const int y = x - __ldg(a.tile_prefix + s);
        g = y / tps;
        tile = y % tps;
    }
    __device__ __forceinline__ void next(const MxArgs &a) {
        if (++tile < tps) return;
        tile = 0;
        if (++g < a.n_kv) return;
        g = 0;
        do {
            if (++s == a.batch) {
                s = 0;
                ++lr;
            }
            N = __ldg(a.lens + s);
            tps = tiles_of(a, s, N);
        } while (tps == 0);
    }
    __device__ __forceinline__ int unit(const MxArgs &a) const { return (lr * a.batch + s) * a.n_kv + g; }
    __device__ __forceinline__ bool last_of_unit() const { return tile == tps - 1; }
};

// tile_prefix[s] = n_kv * (tiles of sequences before s); tile_prefix[batch] = tiles of a layer.
__global__ void tri_mx_prefix_kernel(const MxArgs a) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int run = 0;
    for (int s = 0; s < a.batch; ++s) {
        a.tile_prefix[s] = run;
        run += a.n_kv * MxWalk::tiles_of(a, s, __ldg(a.lens + s));
    }
    a.tile_prefix[a.batch] = run;
}

// phase[s][j][f] = e^{i omega_f (t_s + delta_j)} in fp64.
__global__ void tri_mx_phase_kernel(const MxArgs a, int F) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long n = (long long)a.batch * a.n_off * F;
    if (i >= n) return;
    const int f = (int)(i % F);
    const int j = (int)((i / F) % a.n_off);
    const int s = (int)(i / ((long long)F * a.n_off));
    const long long arg = (long long)__ldg(a.t + s) + a.offsets[j];
    double sn, c;
    sincos(a.omega[f] * (double)arg, &sn, &c);
    a.phase[i] = make_double2(c, sn);
}

// Byte offset of element (row n, dim) of a K-major operand stored as d/64 chunks of
// nrows x 128-byte rows in the 128-byte swizzle (16-byte piece index XOR row % 8).
__host__ __device__ inline unsigned mx_swz_offset(int n, int dim, int nrows) {
    const int c = dim >> 6;
    const unsigned b = (unsigned)(dim & 63) * 2u;
    return (unsigned)c * nrows * 128u + (unsigned)(n >> 3) * 1024u + (unsigned)(n & 7) * 128u +
           ((((b >> 4) ^ (unsigned)(n & 7)) << 4) | (b & 15u));
}

// Coefficient image of every unit: hi and lo bf16 halves, then the norm weights.
template <int D, int G, int LAYOUT>
__global__ void __launch_bounds__(256) tri_mx_image_kernel(const MxArgs a) {
    constexpr int F = D / 2;
    const int unit = blockIdx.x;
    const int g = unit % a.n_kv;
    const int s = (unit / a.n_kv) % a.batch;
    const int lr = unit / (a.n_kv * a.batch);
    const int layer = a.layer_begin + lr;
    const int Hq = a.n_kv * G;
    const int ncol = a.ncol;
    const unsigned half = mx_half_bytes(D, ncol);
    unsigned char *img = a.image + (size_t)unit * mx_image_bytes(D, G, ncol);
    __nv_bfloat16 *hi = reinterpret_cast<__nv_bfloat16 *>(img);
    __nv_bfloat16 *lo = reinterpret_cast<__nv_bfloat16 *>(img + half);
    for (int idx = threadIdx.x; idx < ncol * F; idx += blockDim.x) {
        const int n = idx / F, f = idx % F;
        double re = 0.0, im = 0.0;
        if (n < G * a.noffp) {
            const int h = n / a.noffp, j = min(n % a.noffp, a.n_off - 1);
            const double2 q = a.qbar[((size_t)layer * Hq + (size_t)g * G + h) * F + f];
            const double2 e = a.phase[((size_t)s * a.n_off + j) * F + f];
            re = q.x * e.x - q.y * e.y;
            im = q.x * e.y + q.y * e.x;
        }
        const int dre = LAYOUT == 0 ? f : 2 * f;
        const int dim = LAYOUT == 0 ? f + F : 2 * f + 1;
        const __nv_bfloat16 rh = __float2bfloat16_rn((float)re);
        const __nv_bfloat16 ih = __float2bfloat16_rn((float)im);
        const __nv_bfloat16 rl = __float2bfloat16_rn((float)(re - (double)__bfloat162float(rh)));
        const __nv_bfloat16 il = __float2bfloat16_rn((float)(im - (double)__bfloat162float(ih)));
        if (a.noffp == 1) {
            // one operand of 2 ncol rows per chunk: hi rows, then lo rows (a single MMA reads both)
            hi[mx_swz_offset(n, dre, 2 * ncol) / 2u] = rh;
            hi[mx_swz_offset(n, dim, 2 * ncol) / 2u] = ih;
            hi[mx_swz_offset(ncol + n, dre, 2 * ncol) / 2u] = rl;
            hi[mx_swz_offset(ncol + n, dim, 2 * ncol) / 2u] = il;
        } else {
            const unsigned ore = mx_swz_offset(n, dre, ncol) / 2u, oim = mx_swz_offset(n, dim, ncol) / 2u;
            hi[ore] = rh;
            hi[oim] = ih;
            lo[ore] = rl;
            lo[oim] = il;
        }
    }
    float *w = reinterpret_cast<float *>(img + 2u * half);
    for (int idx = threadIdx.x; idx < G * F; idx += blockDim.x) {
        const int h = idx / F, f = idx % F;
        w[idx] = a.w[((size_t)layer * Hq + (size_t)g * G + h) * F + f];
    }
}

// Shared-memory layout of the scoring kernel (offsets from a 1024-byte aligned base).
struct MxLayout {
    unsigned stage, image, bars, total;
};

__host__ __device__ inline MxLayout mx_layout(int D, int G, int ncol, int nst) {
    MxLayout L;
    const unsigned stage_bytes = (unsigned)(D / 64) * kMxChunkBytes;
    L.stage = 0;
    L.image = (unsigned)nst * stage_bytes;
    L.bars = L.image + 2u * mx_image_bytes(D, G, ncol);
    // full[nst], empty[nst], bfull[2], bempty[2], accfull[kMxMaxAcc], accempty[kMxMaxAcc], TMEM
    // address, abort flag
    L.total = L.bars + (unsigned)(2 * nst + 4 + 2 * kMxMaxAcc) * 8u + 16u + 1024u;  // + alignment slack
    return L;
}

// ---------------------------------------------------------------------------------
// The scoring kernel. NOFF: columns per head (mx_noff_pad of the offset count).
// ---------------------------------------------------------------------------------
template <int D, int G, int LAYOUT, int NOFF>
__global__ void __launch_bounds__(mx_threads(G, NOFF), 1) tri_mx_score_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                     const MxArgs a) {
    constexpr int F = D / 2;
    constexpr int KCH = D / 64;         // 64-dim chunks (128-byte rows)
    constexpr int KSTEPS = D / 16;      // MMA k-steps per tile
    constexpr int NCOL = mx_ncol(G, NOFF);
    // one column per head: hi and lo coefficients form one operand of 2 NCOL rows, so one MMA
    // per k-step reads the key tile once; the epilogue adds the two halves of the accumulator
    constexpr bool CAT = NOFF == 1;
    constexpr int NMMA = CAT ? 2 * NCOL : NCOL;
    constexpr int ACC = mx_acc_cols(NMMA);
    constexpr int NACC = mx_nacc(ACC);
    constexpr int NE = mx_epi_groups(ACC);
    constexpr bool EARLY = NACC >= 2 * NE;                // the MMA warp can run a tile ahead
    constexpr int NCH = CAT ? 0 : (G * NOFF + 31) / 32;  // 32-column chunks of the max
    constexpr int REAL = G * NOFF;      // columns that hold a (head, offset) score
    static_assert(NACC % NE == 0 && NACC * ACC <= 512, "accumulator buffers");
    static_assert(NACC <= kMxMaxAcc, "the barrier block holds kMxMaxAcc accumulator buffers");
    constexpr unsigned kStageBytes = KCH * kMxChunkBytes;
    extern __shared__ unsigned char mx_smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(mx_smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    const int nst = a.nst;
    const MxLayout Ly = mx_layout(D, G, NCOL, nst);
    const unsigned img_bytes = mx_image_bytes(D, G, NCOL);
    const unsigned half = mx_half_bytes(D, NCOL);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Ly.bars);
    uint64_t *empty = full + nst;
    uint64_t *bfull = empty + nst;
    uint64_t *bempty = bfull + 2;
    uint64_t *accfull = bempty + 2;
    uint64_t *accempty = accfull + kMxMaxAcc;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(accempty + kMxMaxAcc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the fused select/compaction over these scores may be launched now (it waits for this grid's
    // completion before it reads a score or takes a unit); its unit counter starts from zero
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (blockIdx.x == 0 && tid == 0) *a.unit_next = 0u;

    // this CTA's tile range
    const int per_layer = __ldg(a.tile_prefix + a.batch);
    const long long total = (long long)per_layer * a.n_layers;
    const long long T0 = total * blockIdx.x / gridDim.x;
    const long long T1 = total * (blockIdx.x + 1) / gridDim.x;
    const int count = (int)(T1 - T0);
    if (count <= 0) return;  // uniform over the CTA, before any barrier or TMEM use

    if (tid == 0) {
        for (int i = 0; i < nst; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 4);  // the 4 warps of the warpgroup that took the tile
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bfull + i, 1);
            mbar_init(bempty + i, 1 + 4 * NE);  // the MMA warp's commit and every epilogue warp
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(accfull + i, 1);
            mbar_init(accempty + i, 4);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    // a TMEM allocation is a power of two of at least 32 columns
    constexpr unsigned kTmemCols = NACC * ACC <= 32 ? 32u : NACC * ACC <= 64 ? 64u : NACC * ACC <= 128 ? 128u
                                                          : NACC * ACC <= 256 ? 256u : 512u;
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    // A wait that ran out ends the CTA's work: every unit its tile range touches is marked, so
    // that the next kernel leaves all of them untouched (their scores may be incomplete).
    auto fail = [&](int unit) {
        record_status(a.status, kDevTimeout, a.unit_base + unit);
        *abort_flag = 1;
        MxWalk w2;
        w2.start(a, T0, per_layer);
        int last = -1;
        for (int k = 0; k < count; ++k) {
            const int u = w2.unit(a);
            if (u != last) {
                atomicExch(a.unit_fail + u, 1);
                last = u;
            }
            if (k + 1 < count) w2.next(a);
        }
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            MxWalk wk;
            wk.start(a, T0, per_layer);
            int seg = -1, prev_unit = -1;
            int issued = 0;
            for (int k = 0; k < count; ++k) {
                if (*abort_flag) break;
                const int unit = wk.unit(a);
                const int stage = k % nst;
                if (k >= nst && !mbar_wait_bounded(empty + stage, (unsigned)((k / nst - 1) & 1), a.wait_tries)) {
                    fail(unit);
                    break;
                }
                if (unit != prev_unit) {
                    ++seg;
                    prev_unit = unit;
                    const int ub = seg & 1;
                    if (seg >= 2 && !mbar_wait_bounded(bempty + ub, (unsigned)((seg / 2 - 1) & 1), a.wait_tries)) {
                        fail(unit);
                        break;
                    }
                    fence_proxy_async_smem();
                    mbar_expect_tx(bfull + ub, img_bytes);
                    tma_load_1d(smem + Ly.image + ub * img_bytes, a.image + (size_t)unit * img_bytes, img_bytes,
                                bfull + ub, policy_evict_last());
                }
                // key rows of this tile, one TMA box of piece_rows rows per 64-dim chunk; boxes past
                // the unit's length or on an unallocated page are not loaded
                const int pr = a.piece_rows;
                const int n_pieces = kMxTile / pr;
                unsigned bytes = 0;
                for (int p = 0; p < n_pieces; ++p) {
                    const int r0 = wk.tile * kMxTile + p * pr;
                    if (r0 >= wk.N) break;
                    if (a.paged) {
                        const int pg = __ldg(a.block_table + (long long)wk.s * a.max_pages + r0 / a.page_size);
                        if (pg < 0 || pg >= a.n_pages) continue;
                    }
                    bytes += (unsigned)KCH * pr * 128u;
                }
                fence_proxy_async_smem();
                mbar_expect_tx(full + stage, bytes);
                unsigned char *dst = smem + Ly.stage + (unsigned)stage * kStageBytes;
                // test hook: the unit's first tile is armed but never loaded, so its wait runs out
                const bool withhold = wk.tile == 0 && a.unit_base + unit == a.inject_unit;
                for (int p = 0; p < (withhold ? 0 : n_pieces); ++p) {
                    const int r0 = wk.tile * kMxTile + p * pr;
                    if (r0 >= wk.N) break;
                    long long row;
                    if (a.paged) {
                        const int pg = __ldg(a.block_table + (long long)wk.s * a.max_pages + r0 / a.page_size);
                        if (pg < 0 || pg >= a.n_pages) continue;
                        row = (((long long)wk.lr * a.n_pages + pg) * a.n_kv + wk.g) * (long long)a.page_size +
                              (r0 % a.page_size);
                    } else {
                        row = (((long long)wk.lr * a.batch + wk.s) * a.n_kv + wk.g) * (long long)a.cap_u + r0;
                    }
#pragma unroll
                    for (int c = 0; c < KCH; ++c)
                        tma_load_2d(dst + c * kMxChunkBytes + (unsigned)p * pr * 128u, &tmap, c * 64, (int)row,
                                    full + stage, pol);
                }
                ++issued;
                if (k + 1 < count) wk.next(a);
            }
            // copies still in flight must land before the CTA exits
            for (int k = (issued > nst ? issued - nst : 0); k < issued; ++k)
                (void)mbar_wait_bounded(full + k % nst, (unsigned)((k / nst) & 1), a.wait_tries);
            for (int sg = (seg > 1 ? seg - 1 : 0); sg <= seg; ++sg)
                (void)mbar_wait_bounded(bfull + (sg & 1), (unsigned)((sg / 2) & 1), a.wait_tries);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = mx_idesc(NMMA);
            MxWalk wk;
            wk.start(a, T0, per_layer);
            int seg = -1, prev_unit = -1;
            int issued = 0;
            for (int k = 0; k < count; ++k) {
                if (*abort_flag) break;
                const int unit = wk.unit(a);
                const int stage = k % nst;
                if (unit != prev_unit) {
                    ++seg;
                    prev_unit = unit;
                    if (!mbar_wait_bounded(bfull + (seg & 1), (unsigned)((seg / 2) & 1), a.wait_tries)) {
                        fail(unit);
                        break;
                    }
                }
                const int ab = k % NACC;
                if (k >= NACC && !mbar_wait_bounded(accempty + ab, (unsigned)((k / NACC - 1) & 1), a.wait_tries)) {
                    fail(unit);
                    break;
                }
                if (!mbar_wait_bounded(full + stage, (unsigned)((k / nst) & 1), a.wait_tries)) {
                    fail(unit);
                    break;
                }
                tc_fence_after();
                const unsigned char *As = smem + Ly.stage + (unsigned)stage * kStageBytes;
                const unsigned char *Bs = smem + Ly.image + (seg & 1) * img_bytes;
                const uint32_t dt = tmem_base + (uint32_t)(ab * ACC);
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ++ks) {
                    const unsigned koff = (unsigned)(ks & 3) * 32u;  // K = 16 bf16 = 32 bytes per step
                    const uint64_t ad = mx_desc(As + (ks >> 2) * kMxChunkBytes + koff);
                    if constexpr (CAT) {
                        const uint64_t bc = mx_desc(Bs + (unsigned)(ks >> 2) * NMMA * 128u + koff);
                        mx_mma(dt, ad, bc, idesc, ks > 0 ? 1 : 0);
                    } else {
                        const uint64_t bh = mx_desc(Bs + (unsigned)(ks >> 2) * NCOL * 128u + koff);
                        const uint64_t bl = mx_desc(Bs + half + (unsigned)(ks >> 2) * NCOL * 128u + koff);
                        mx_mma(dt, ad, bh, idesc, ks > 0 ? 1 : 0);
                        mx_mma(dt, ad, bl, idesc, 1);
                    }
                }
                mx_commit(accfull + ab);
                if (k + 1 == count || wk.last_of_unit()) mx_commit(bempty + (seg & 1));
                ++issued;
                if (k + 1 < count) wk.next(a);
            }
            // every MMA issued must have completed before the TMEM is released
            if (issued > 0)
                (void)mbar_wait_bounded(accfull + (issued - 1) % NACC, (unsigned)(((issued - 1) / NACC) & 1),
                                        a.wait_tries);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: warpgroup wg takes tiles k = wg (mod NE) ----------------
        const int ew = warp - 2;
        const int wg = ew >> 2;
        const int q = warp & 3;       // TMEM lane quarter this warp may access
        const int r = q * 32 + lane;  // key row within the tile
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const unsigned rowoff = (unsigned)(r >> 3) * 1024u + (unsigned)(r & 7) * 128u;
        MxWalk wk;
        wk.start(a, T0, per_layer);
        int seg = -1, prev_unit = -1;
        for (int k = 0; k < count; ++k) {
            if (*abort_flag) break;
            const int unit = wk.unit(a);
            if (unit != prev_unit) {
                ++seg;
                prev_unit = unit;
            }
            const bool seg_end = k + 1 == count || wk.last_of_unit();
            if (k % NE == wg) {
                const int stage = k % nst;
                const int ab = k % NACC;
                // norm score first: it needs only the key rows, which usually land before the
                // tile's MMAs finish, so this work overlaps them
                const bool ok_st =
                    __all_sync(0xffffffffu, mbar_wait_bounded(full + stage, (unsigned)((k / nst) & 1), a.wait_tries));
                const bool ok_b = __all_sync(
                    0xffffffffu, mbar_wait_bounded(bfull + (seg & 1), (unsigned)((seg / 2) & 1), a.wait_tries));
                if (!ok_st || !ok_b) {
                    if (lane == 0) fail(unit);
                    break;
                }
                const uint32_t tbase = tmem_base + lane_base + (uint32_t)(ab * ACC);
                // accumulator columns are read in chunks of 32, each chunk's load issued before the
                // previous chunk is reduced; one column per head takes 8 hi and 8 lo columns
                uint32_t acc_hi[8], acc_lo[8];
                uint32_t pa[16], pb[16], qa[16], qb[16];
                auto issue_chunk = [&](int c, uint32_t(&x)[16], uint32_t(&y)[16]) {
                    tmem_ld16_issue(tbase + (uint32_t)(32 * c), x);
                    if (32 * c + 16 < REAL) tmem_ld16_issue(tbase + (uint32_t)(32 * c + 16), y);
                };
                auto issue_first = [&]() {
                    if constexpr (CAT) {
                        tmem_ld8_issue(tbase, acc_hi);
                        tmem_ld8_issue(tbase + (uint32_t)NCOL, acc_lo);
                    } else {
                        issue_chunk(0, pa, pb);
                    }
                };
                // where the MMA warp runs a tile ahead of this warpgroup (two accumulators each), the
                // accumulator is usually complete by now, and its first chunk is read while the norm
                // term is computed; otherwise the norm term overlaps the tile's MMAs instead
                if constexpr (EARLY) {
                    const bool ok_acc0 = __all_sync(
                        0xffffffffu, mbar_wait_bounded(accfull + ab, (unsigned)((k / NACC) & 1), a.wait_tries));
                    if (!ok_acc0) {
                        if (lane == 0) fail(unit);
                        break;
                    }
                    tc_fence_after();
                    issue_first();
                }
                const unsigned char *As = smem + Ly.stage + (unsigned)stage * kStageBytes;
                const float *wsm =
                    reinterpret_cast<const float *>(smem + Ly.image + (seg & 1) * img_bytes + 2u * half);
                auto piece = [&](int dim) {  // 8 dims starting at dim (a multiple of 8)
                    const unsigned off = (unsigned)(dim >> 6) * kMxChunkBytes + rowoff +
                                         ((((unsigned)(dim & 63) >> 3) ^ (unsigned)(r & 7)) << 4);
                    return *reinterpret_cast<const uint4 *>(As + off);
                };
                float2 nrm[G];
#pragma unroll
                for (int h = 0; h < G; ++h) nrm[h] = make_float2(0.f, 0.f);
#pragma unroll 2
                for (int f0 = 0; f0 < F; f0 += 8) {
                    // band moduli of bands f0 .. f0 + 7, as four pairs (f, f + 1)
                    float2 nb[4];
                    if (LAYOUT == 0) {
                        const uint4 xr = piece(f0), xi = piece(F + f0);
                        const unsigned wr[4] = {xr.x, xr.y, xr.z, xr.w}, wi[4] = {xi.x, xi.y, xi.z, xi.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 re = make_float2(bf16lo(wr[e]), bf16hi(wr[e]));
                            const float2 im = make_float2(bf16lo(wi[e]), bf16hi(wi[e]));
                            const float2 sq = __ffma2_rn(im, im, __fmul2_rn(re, re));
                            nb[e] = make_float2(sqrt_approx(sq.x), sqrt_approx(sq.y));
                        }
                    } else {
                        const uint4 x0 = piece(2 * f0), x1 = piece(2 * f0 + 8);
                        const unsigned wv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 re = make_float2(bf16lo(wv[2 * e]), bf16lo(wv[2 * e + 1]));
                            const float2 im = make_float2(bf16hi(wv[2 * e]), bf16hi(wv[2 * e + 1]));
                            const float2 sq = __ffma2_rn(im, im, __fmul2_rn(re, re));
                            nb[e] = make_float2(sqrt_approx(sq.x), sqrt_approx(sq.y));
                        }
                    }
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float4 w0 = *reinterpret_cast<const float4 *>(wsm + h * F + f0);
                        const float4 w1 = *reinterpret_cast<const float4 *>(wsm + h * F + f0 + 4);
                        nrm[h] = __ffma2_rn(make_float2(w0.x, w0.y), nb[0], nrm[h]);
                        nrm[h] = __ffma2_rn(make_float2(w0.z, w0.w), nb[1], nrm[h]);
                        nrm[h] = __ffma2_rn(make_float2(w1.x, w1.y), nb[2], nrm[h]);
                        nrm[h] = __ffma2_rn(make_float2(w1.z, w1.w), nb[3], nrm[h]);
                    }
                }

                if constexpr (!EARLY) {
                    const bool ok_acc = __all_sync(
                        0xffffffffu, mbar_wait_bounded(accfull + ab, (unsigned)((k / NACC) & 1), a.wait_tries));
                    if (!ok_acc) {
                        if (lane == 0) fail(unit);
                        break;
                    }
                    tc_fence_after();
                    issue_first();
                }
                // max over each head's NOFF columns
                float best[G];
#pragma unroll
                for (int h = 0; h < G; ++h) best[h] = __int_as_float(0xff800000);
                if constexpr (CAT) {
                    // columns [0, G): the hi products, [NCOL, NCOL + G): the lo products
                    tmem_wait_ld8(acc_hi, acc_lo);
#pragma unroll
                    for (int h = 0; h < G; ++h) best[h] = __uint_as_float(acc_hi[h]) + __uint_as_float(acc_lo[h]);
                }
                auto reduce_chunk = [&](int c, const uint32_t(&v0)[16], const uint32_t(&v1)[16]) {
                    // columns pair up within a head (offsets 2j, 2j + 1) for one three-input max;
                    // every index below is a compile-time constant once the loops unroll
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int col = 32 * c + i;
                        if (col < REAL) {
                            const int h = col / NOFF, j = col - h * NOFF;
                            const float x = __uint_as_float(i < 16 ? v0[i] : v1[i - 16]);
                            const bool first = (j % 2 == 0) && j + 1 < NOFF && i + 1 < 32 && col + 1 < REAL;
                            const bool second = (j % 2 == 1) && i > 0;
                            if (first) {
                                const float y = __uint_as_float(i + 1 < 16 ? v0[i + 1] : v1[i + 1 - 16]);
                                best[h] = max3f(best[h], x, y);
                            } else if (!second) {
                                best[h] = fmaxf(best[h], x);
                            }
                        }
                    }
                };
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const bool two = 32 * c + 16 < REAL;
                    if (c % 2 == 0) {
                        tmem_wait_ld(pa);
                        if (two) tmem_after_wait(pb);
                        if (c + 1 < NCH) issue_chunk(c + 1, qa, qb);
                        reduce_chunk(c, pa, pb);
                    } else {
                        tmem_wait_ld(qa);
                        if (two) tmem_after_wait(qb);
                        if (c + 1 < NCH) issue_chunk(c + 1, pa, pb);
                        reduce_chunk(c, qa, qb);
                    }
                }
                tc_fence_before();
                __syncwarp();
                // the MMA has finished with the key tile and the accumulator: release both
                if (lane == 0) {
                    mbar_arrive(accempty + ab);
                    mbar_arrive(empty + stage);
                }
                const int key = wk.tile * kMxTile + r;
                const bool valid = key < wk.N;
                float sv[G];
#pragma unroll
                for (int h = 0; h < G; ++h) sv[h] = best[h] + (nrm[h].x + nrm[h].y);
                if (valid) {
                    float *dst = a.pre + ((long long)unit * a.cap_u + key) * G;
                    if constexpr (G >= 4) {
#pragma unroll
                        for (int h4 = 0; h4 < G; h4 += 4)
                            *reinterpret_cast<float4 *>(dst + h4) =
                                make_float4(sv[h4], sv[h4 + 1], sv[h4 + 2], sv[h4 + 3]);
                    } else if constexpr (G == 2) {
                        *reinterpret_cast<float2 *>(dst) = make_float2(sv[0], sv[1]);
                    } else {
                        dst[0] = sv[0];
                    }
                }
            }
            if (seg_end) {
                // every tile of this warp's warpgroup in the unit is done: release the unit's
                // coefficient image (after its load completed, so that this arrival can only
                // count toward this unit's use of the buffer)
                const bool ok_b = __all_sync(
                    0xffffffffu, mbar_wait_bounded(bfull + (seg & 1), (unsigned)((seg / 2) & 1), a.wait_tries));
                if (!ok_b) {
                    if (lane == 0) fail(unit);
                    break;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bempty + (seg & 1));
            }
            if (k + 1 < count) wk.next(a);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace tri
