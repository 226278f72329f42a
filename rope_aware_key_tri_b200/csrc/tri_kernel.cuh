// tri_kernel.cuh -- the fused TriAttention scoring-and-pruning kernel for sm_100a.
//
// Pages cited (titles; sections as headed on each page):
//   [Deep-dive]  "TriAttention深度解析：用三角函数革命性压缩KV Cache，让长推理从「显存地狱」中脱困"
//   [Stage]      "旋转舞台上的追光者——TriAttention如何用三角函数破解长文本推理的内存困局"
//   [10100]      the 10100.com article 127765992 on TriAttention
//   [Summary]    "TriAttention：面向长文本推理的高效KV缓存压缩，2.5倍吞吐提升与10.7倍内存缩减"
//
// A persistent grid of thread-block clusters (two CTAs per SM) walks the units; one
// cluster of cs CTAs owns one unit (sequence s, layer l, KV head g) at a time and runs
// the whole pass on it:
//
//   prologue  C_{h,f} = (qbar_{h,f} A_f) e^{i omega_f t}, with A_f = mean_delta e^{i omega_f delta}
//             (fp64 phase, rounded to fp32 once). Because the stored key is post-RoPE,
//             mean_delta |qbar_f||k_f| cos(omega_f (t+delta-p) + arg qbar_f - arg k_f)
//             = Re(C_f conj(k~_f)), so the trigonometric series of [Stage]
//             §TriAttention：把理论变成算法 item 1, averaged over the offsets of [Deep-dive] §3.3,
//             becomes one dot product per key and head; positions drop out.
//   score     per key: s_h = sum_j c_{h,j} k~_j + sum_f w_{h,f} |k~_f|, w = (1 - R) E|q|
//             ([Stage] item 2 with the (1 - R) weight of [10100] §TriAttention方法). Keys
//             stream from HBM by TMA bulk copies (cp.async.bulk, mbarrier completion,
//             evict-first L2 hint) into per-warp buffers; each key is split over LPK lanes,
//             every lane keeps its slice of the coefficients in registers and accumulates
//             with packed fp32x2 FMAs; a reduce-scatter over the lanes finishes the G heads.
//             Scores go to a per-cluster scratch slot with an evict-last L2 hint, so they
//             are re-read from L2, not HBM.
//   z / max   per head: mean and population std over all of the unit's keys (fp64 sums
//             exchanged between the cluster's CTAs through distributed shared memory),
//             z = (s - mu) / sigma (0 for a flat head), max over the G heads
//             ([10100] §TriAttention方法; [Summary] §方案设计 item 4).
//   select    top-B by max-z: up to four 8-bit radix passes over an order-preserving
//             uint32 image of the fp32 value, histograms merged across the cluster; exact
//             ties at the threshold go to the lower slot.
//   compact   in-place stable gather of the kept K/V/position rows to slots [0, B)
//             ([Deep-dive] §4 prune_kv_cache: top-k then sort). Destinations are taken in
//             rounds in ascending order; in each round every CTA first copies its
//             sources into shared memory (cp.async), then writes them. A kept row never
//             moves to a higher slot, so no round overwrites a row that a later round still
//             has to read; only the rows that come from below slot B can be overwritten
//             by another CTA's writes of the same round, and their rounds put a cluster
//             barrier between the reads and the writes.
#pragma once

#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tri {

namespace cg = cooperative_groups;

constexpr int kStageRows = 16;      // rows per TMA bulk copy (one copy never crosses a page)
constexpr int kBins = 256;          // radix digit width: 8 bits
// Warps per CTA (two CTAs per SM). A lane keeps 48 coefficients in registers with 8 warps
// (128 registers per thread) and 96 with 6 warps (168); GQA 8 needs the latter. The variant that
// reads precomputed scores (pre) holds no coefficients and always runs 8 warps.
__host__ __device__ constexpr int cta_warps(int G, bool pre = false) { return (G >= 8 && !pre) ? 6 : 8; }
__host__ __device__ constexpr int cta_threads(int G, bool pre = false) { return cta_warps(G, pre) * 32; }
constexpr int kMinBlocks = 2;
constexpr int kMaxCluster = 16;
constexpr int kModePrune = 0;
constexpr int kModeScore = 1;
constexpr int kDevLenGtCap = 1;
constexpr int kDevBadPage = 2;
constexpr int kDevTimeout = 3;
constexpr int kDevInternal = 4;
constexpr int kDevTNotAfterPos = 5;
constexpr int kWaitTries = 1024;             // bounded mbarrier waits (the default number of tries) ...
constexpr unsigned kWaitSuspendNs = 1000000; // ... each suspending the warp for up to 1 ms

struct Args {
    uint16_t *K;                 // bf16 bits
    uint16_t *V;
    int32_t *pos;
    const int32_t *lens;
    int32_t *lens_out;
    const int32_t *block_table;
    const int32_t *t;
    int batch, n_kv, cap_u;
    int paged, page_size, max_pages, n_pages;
    int page_shift;              // log2(page_size) when a power of two, else -1
    int layer_begin;
    int budget;
    int n_units;
    const double *omega;         // [F]
    const double2 *Qc;           // [L][Hq][F]  qbar * A
    const float *w;              // [L][Hq][F]  (1 - R) E|q|
    float *raw;                  // score mode outputs (or null)
    float *zmax;
    int mode;
    int cs;                      // cluster size (CTAs per unit)
    int kpc_max;                 // key capacity of one CTA (multiple of 32)
    int ring_extra;              // staging bytes appended to the TMA ring
    int nslot;                   // TMA buffers per warp
    float *scratch;              // per-cluster slots: [cap_u][G] scores then [cap_u] order keys
    long long slot_floats;       // floats per slot
    unsigned long long *status;  // first device-detected problem
    unsigned int *counter;       // completed-CTA counter (last CTA updates lens_out)
    unsigned int *unit_next;     // dynamic unit assignment: the next free unit; zeroed by the
                                 // kernel launched just before (validation or tensor-core scoring)
    int32_t *seq_bad;            // [batch] the validation kernel's verdicts (0: accepted)
    const float *pre;            // precomputed scores [n_units][cap_u][G] (tensor-core engine)
    const int32_t *unit_fail;    // [n_units] units whose precomputed scores are missing
    long long unit_base;         // added to the unit index in device status reports
    int wait_tries;              // tries (about 1 ms each) of every bounded wait
    long long inject_unit;       // test hook: the unit whose first key copy is withheld (-1: none)
    int stagger;                 // 1: clusters holding one unit fewer start half a unit period late
    unsigned *fail_count;        // units left uncompacted by a unit-level failure ...
    int32_t *fail_units;         // ... and the first fail_cap of them
    int fail_cap;
};

// Per-CTA values other CTAs of the cluster read through distributed shared memory.
struct Xch {
    double sum[8];
    double m2[8];
    float mn[8];
    float mx[8];
    int ties;
    int fail;
    int next[2];  // rank 0: the cluster's next units under dynamic assignment (by parity)
};

struct Layout {
    unsigned ring, coef_t, coef_w, phase, whist, bhist, ghist, lmask, gmask, gpre, xch, misc,
        srcidx, bars, total;
    int stage_rows;    // compaction rows per CTA per round (staged in the ring)
    unsigned ring_bytes;  // the TMA ring plus the extra staging the compaction may use
};

__host__ __device__ inline unsigned align_up(unsigned x, unsigned a) { return (x + a - 1) / a * a; }

// extra: bytes appended to the TMA ring where shared memory is left over; the order keys and
// the compaction's staging use the whole region, the key stream only the ring.
__host__ __device__ inline Layout make_layout(int D, int G, int nslot, int kpc, int cs, int extra,
                                              bool pre = false) {
    const int kWarps = cta_warps(G, pre);
    Layout L;
    unsigned o = 0;
    const int F = D / 2;
    const int nwl = kpc / 32;
    L.ring = o;
    o = align_up(o + (unsigned)kWarps * nslot * kStageRows * D * 2u + (unsigned)extra, 128);
    L.ring_bytes = o;
    const unsigned row_bytes = (unsigned)D * 2u * 2u + 4u;
    int S = (int)(o / row_bytes);
    S = S / 16 * 16;
    L.stage_rows = S;
    L.coef_t = o;
    o = align_up(o + (unsigned)G * D * 4u, 16);
    L.coef_w = o;
    o = align_up(o + (unsigned)G * F * 4u, 16);
    L.phase = o;
    o = align_up(o + (unsigned)F * 16u, 16);
    L.whist = o;
    o = align_up(o + (unsigned)kWarps * kBins * 4u, 16);
    L.bhist = o;
    o = align_up(o + 2u * kBins * 4u, 16);
    L.ghist = o;
    o = align_up(o + (unsigned)kBins * 4u, 16);
    L.lmask = o;
    o = align_up(o + (unsigned)nwl * 4u, 16);
    L.gmask = o;
    o = align_up(o + (unsigned)cs * nwl * 4u, 16);
    L.gpre = o;
    o = align_up(o + ((unsigned)cs * nwl + 1u) * 4u, 16);
    L.xch = o;
    o = align_up(o + sizeof(Xch), 16);
    L.misc = o;  // block-reduction scratch: kWarps + 1 doubles, 64 ints, 32 floats
    o = align_up(o + (unsigned)(kWarps + 1) * 8u + 64u * 4u + 32u * 4u, 16);
    L.srcidx = o;
    o = align_up(o + (unsigned)(S > 0 ? S : 1) * 4u, 16);
    L.bars = o;
    o = align_up(o + (unsigned)kWarps * nslot * 8u, 16);
    L.total = o;
    return L;
}

// ---------------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------------
__device__ __forceinline__ unsigned smem_u32(const void *p) {
    return (unsigned)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// One potentially blocking test of the barrier phase: the hardware suspends the warp until
// the phase completes or the time hint runs out, so waiting costs no issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitSuspendNs)
        : "memory");
    return ok != 0;
}

// Bounded wait (tries x about 1 ms at most): returns false if the phase never completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned parity, int tries) {
    for (int i = 0; i < tries; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 1-D bulk copy global -> shared, completion signalled on an mbarrier, with an L2
// eviction-priority hint (no multicast).
__device__ __forceinline__ void tma_load_1d(void *dst_smem, const void *src_gmem, unsigned bytes,
                                            uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void st_hint(float *p, float v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(policy) : "memory");
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// The staggered start's wait (see the fused kernel); kept out of line, away from the kernel's
// register allocation. Bounded by its own clock and by an iteration count.
__device__ __noinline__ void stagger_wait(int n_units, int n_clusters, int cid, const int32_t *lens, int n_kv,
                                          int batch, int cap_u, int budget, int D) {
    const int q = n_units / n_clusters, r = n_units % n_clusters;
    if (q < 2 || r == 0 || cid < r) return;
    const int N0 = min(max(__ldg(lens + (cid / n_kv) % batch), 0), cap_u);
    const float bytes = (float)N0 * (float)(2 * D) + (float)min(N0, budget) * (float)(8 * D + 8);
    const unsigned long long wait_ns = (unsigned long long)(bytes * (float)n_clusters * (0.5f / 4600.f));
    const unsigned long long t0 = global_ns();
    for (int it = 0; it < (1 << 22) && global_ns() - t0 < wait_ns; ++it) __nanosleep(256);
}

// An int in cluster rank 0's shared memory at the address of *local (this CTA's copy of the
// same variable). Written as asm so that the remote address is formed where it is used, not
// held in registers across a loop.
__device__ __forceinline__ int ld_rank0_int(const int *local) {
    const unsigned laddr = (unsigned)__cvta_generic_to_shared(local);
    unsigned raddr;
    int v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(raddr) : "r"(laddr));
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(raddr) : "memory");
    return v;
}

__device__ __forceinline__ void prefetch_l1(const void *p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async4(void *dst_smem, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}

// Band modulus. Denormal squared norms (below 1.2e-38) flush to zero, which moves a score by
// less than 1e-19; the .ftz form is a single MUFU operation.
__device__ __forceinline__ float sqrt_approx(float x) {
    float y;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float bf16lo(unsigned w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(unsigned w) { return __uint_as_float(w & 0xffff0000u); }

// Order-preserving map of an fp32 value onto uint32 (larger float -> larger integer).
__device__ __forceinline__ unsigned float_key(float z) {
    unsigned u = __float_as_uint(z);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void record_status(unsigned long long *st, int code, long long unit) {
    unsigned long long v = ((unsigned long long)(unsigned)code << 32) | (unsigned long long)(unsigned)unit;
    atomicCAS(st, 0ull, v);
}

// A unit-level failure: the unit is left uncompacted (its first min(len, B) slots keep their
// original rows), the status word records the first problem, and the unit joins the list the
// host reads with tri_get_failed_units.
__device__ __forceinline__ void record_unit_failure(unsigned long long *st, unsigned *fail_count,
                                                    int32_t *fail_units, int fail_cap, int code, long long unit) {
    record_status(st, code, unit);
    if (fail_count) {
        const unsigned k = atomicAdd(fail_count, 1u);
        if ((int)k < fail_cap) fail_units[k] = (int32_t)unit;
    }
}

// Row index (in rows of head_dim elements) of logical slot i of a unit.
__device__ __forceinline__ long long row_of(const Args &a, int lr, int s, int g, int i) {
    if (!a.paged) return (((long long)lr * a.batch + s) * a.n_kv + g) * (long long)a.cap_u + i;
    // a row address per moved row and lane: shifts for the usual power-of-two page sizes
    int pi, po;
    if (a.page_shift >= 0) {
        pi = i >> a.page_shift;
        po = i & (a.page_size - 1);
    } else {
        pi = i / a.page_size;
        po = i - pi * a.page_size;
    }
    const int page = __ldg(a.block_table + (long long)s * a.max_pages + pi);
    return (((long long)lr * a.n_pages + page) * a.n_kv + g) * (long long)a.page_size + po;
}

// k-th (0-based) set bit of m.
__device__ __forceinline__ int select_bit(unsigned m, int k) {
    int pos = 0;
#pragma unroll
    for (int sh = 16; sh >= 1; sh >>= 1) {
        const unsigned low = m & ((1u << sh) - 1u);
        const int c = __popc(low);
        if (k >= c) {
            k -= c;
            m >>= sh;
            pos += sh;
        } else {
            m = low;
        }
    }
    return pos;
}

// Exclusive scan of n ints in place in shared memory (any n); returns the total.
// All threads of the block must call it.
template <int kWarps>
__device__ int block_exclusive_scan(int *a, int n, int *scratch /* kWarps + 2 ints */) {
    constexpr int kThreads = kWarps * 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int PER = 4;
    int carry = 0;
    for (int base = 0; base < n; base += PER * kThreads) {
        int v[PER];
        int local = 0;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int i = base + tid * PER + k;
            v[k] = i < n ? a[i] : 0;
            local += v[k];
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) scratch[warp] = incl;
        __syncthreads();
        if (tid == 0) {
            int run = 0;
            for (int w = 0; w < kWarps; ++w) {
                const int x = scratch[w];
                scratch[w] = run;
                run += x;
            }
            scratch[kWarps] = run;
        }
        __syncthreads();
        int ex = carry + scratch[warp] + incl - local;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int i = base + tid * PER + k;
            if (i < n) a[i] = ex;
            ex += v[k];
        }
        carry += scratch[kWarps];
        __syncthreads();
    }
    return carry;
}

// ---------------------------------------------------------------------------------
// Sequence-level checks of one call, run before any unit of the call is touched, so that
// every unit of a sequence gets the same verdict: the length within the capacity, every page
// of the sequence inside the pool, and every unit's last cached position below t (positions
// ascend within a unit, so the last one is the largest). One block per sequence;
// seq_bad[s] receives the problem code (0: accepted), which the fused kernel and the
// max-over-offsets scoring kernel read. The first problem also goes to the status word.
// ---------------------------------------------------------------------------------
constexpr int kValidateThreads = 256;

__global__ void __launch_bounds__(kValidateThreads) tri_validate_kernel(const Args a) {
    // the fused kernel may be launched now: it waits for this grid's completion (and memory)
    // before it reads a verdict or takes a unit
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (blockIdx.x == 0 && threadIdx.x == 0 && a.unit_next) *a.unit_next = 0u;
    const int s = blockIdx.x;
    const int N = __ldg(a.lens + s);
    const int n_layers = a.n_units / (a.batch * a.n_kv);
    __shared__ int bad_unit_s;
    if (threadIdx.x == 0) bad_unit_s = 0x7fffffff;
    __syncthreads();
    int code = 0;
    long long unit = (long long)s * a.n_kv;  // the sequence's first unit of the call
    if (N < 0 || N > a.cap_u) {
        code = kDevLenGtCap;
    } else if (N > 0) {  // uniform over the block
        if (a.paged) {
            const int np = (N + a.page_size - 1) / a.page_size;
            int mine = 0;
            for (int p = threadIdx.x; p < np; p += kValidateThreads) {
                const int pg = __ldg(a.block_table + (long long)s * a.max_pages + p);
                if (pg < 0 || pg >= a.n_pages) mine = 1;
            }
            if (__syncthreads_or(mine)) code = kDevBadPage;
        }
        if (!code && a.pos) {
            const int tq = __ldg(a.t + s);
            for (int k = threadIdx.x; k < n_layers * a.n_kv; k += kValidateThreads) {
                const int lr = k / a.n_kv, g = k % a.n_kv;
                if (__ldg(a.pos + row_of(a, lr, s, g, N - 1)) >= tq)
                    atomicMin(&bad_unit_s, (lr * a.batch + s) * a.n_kv + g);
            }
            __syncthreads();
            if (bad_unit_s != 0x7fffffff) {
                code = kDevTNotAfterPos;
                unit = bad_unit_s;
            }
        }
    }
    if (threadIdx.x == 0) {
        a.seq_bad[s] = code;
        if (code) record_status(a.status, code, a.unit_base + unit);
    }
}

// ---------------------------------------------------------------------------------
// Per-key slice geometry. A key of D dims is split over LPK lanes; each lane holds DH
// consecutive dims from the first half of the row and the DH dims D/2 further on, i.e.
// DH whole bands in either rotary layout. DH is chosen so that a lane keeps 3 * DH * G
// (48 with 8 warps, 96 with 6) coefficients in registers: its DH trig coefficients of each half and its DH
// norm weights, for every head of the group.
// ---------------------------------------------------------------------------------
template <int D, int G>
struct Geo {
    static constexpr int DH_REG = (cta_warps(G) == 8 ? 16 : 32) / G;
    static constexpr int DH = DH_REG < D / 4 ? DH_REG : D / 4;  // at least 2 lanes per key
    static constexpr int LPK = D / (2 * DH);
    static constexpr int KPP = 32 / LPK;  // keys per warp per pass
    static constexpr int NP = DH / 2;     // float2 pairs per half-chunk
    static_assert(LPK >= G, "a key needs at least G lanes");
    static_assert(LPK >= 2 && 32 % LPK == 0, "LPK must divide the warp");
    static_assert(KPP <= kStageRows, "a pass must fit in one stage");
    static_assert(DH % 4 == 0, "DH must be a multiple of 4");
};

// Load DH consecutive bf16 from smem as DH/2 32-bit words.
template <int DH>
__device__ __forceinline__ void load_chunk(const uint16_t *p, unsigned (&w)[DH / 2]) {
    if constexpr (DH == 4) {
        const uint2 x = *reinterpret_cast<const uint2 *>(p);
        w[0] = x.x; w[1] = x.y;
    } else {
#pragma unroll
        for (int q = 0; q < DH / 8; ++q) {
            const uint4 x = *reinterpret_cast<const uint4 *>(p + 8 * q);
            w[4 * q] = x.x; w[4 * q + 1] = x.y; w[4 * q + 2] = x.z; w[4 * q + 3] = x.w;
        }
    }
}

// bf16 pairs -> fp32 pairs. Half layout: pair p = dims (2p, 2p+1). Interleaved layout:
// pair 2i = dims (4i, 4i+2), pair 2i+1 = dims (4i+1, 4i+3), so that the two members of
// each rotary band land in matching lanes of two pairs (one fp32x2 square-sum per two bands).
template <int NP, int LAYOUT>
__device__ __forceinline__ void unpack_pairs(const unsigned (&w)[NP], float2 (&x)[NP]) {
    if constexpr (LAYOUT == 0) {
#pragma unroll
        for (int p = 0; p < NP; ++p) x[p] = make_float2(bf16lo(w[p]), bf16hi(w[p]));
    } else {
#pragma unroll
        for (int i = 0; i < NP / 2; ++i) {
            x[2 * i] = make_float2(bf16lo(w[2 * i]), bf16lo(w[2 * i + 1]));
            x[2 * i + 1] = make_float2(bf16hi(w[2 * i]), bf16hi(w[2 * i + 1]));
        }
    }
}

// The G scores of one key (16-byte aligned rows of G floats).
template <int G>
__device__ __forceinline__ void load_scores(const float *p, float (&v)[G]) {
    if constexpr (G >= 4) {
#pragma unroll
        for (int q = 0; q < G / 4; ++q) {
            const float4 x = *reinterpret_cast<const float4 *>(p + 4 * q);
            v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
        }
    } else if constexpr (G == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        v[0] = x.x; v[1] = x.y;
    } else {
        v[0] = *p;
    }
}

// Dim index (within the lane's DH-dim chunk) of element e (0 = .x, 1 = .y) of pair p.
template <int LAYOUT>
__host__ __device__ constexpr int pair_dim(int p, int e) {
    return LAYOUT == 0 ? 2 * p + e : 4 * (p / 2) + (p % 2) + 2 * e;
}

// ---------------------------------------------------------------------------------
// The fused kernel. Grid: n_clusters * cs CTAs (clusters of cs), persistent over units.
// ---------------------------------------------------------------------------------
// PRE: the scores come precomputed (one [cap_u][G] row block per unit) instead of being
// computed here; the z-score, select and compaction are the same.
template <int D, int G, int LAYOUT, bool PRE = false>
__global__ void __launch_bounds__(cta_threads(G, PRE), kMinBlocks) tri_fused_kernel(const Args a) {
    constexpr int kWarps = cta_warps(G, PRE);
    constexpr int kThreads = kWarps * 32;
    constexpr int F = D / 2;
    using GE = Geo<D, G>;
    constexpr int DH = GE::DH;
    constexpr int LPK = GE::LPK;
    constexpr int KPP = GE::KPP;
    constexpr int NP = GE::NP;
    constexpr unsigned FULL = 0xffffffffu;
    constexpr unsigned kStageBytes = kStageRows * D * 2;

    extern __shared__ __align__(128) unsigned char smem[];
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = a.cs;
    const int crank = (int)cluster.block_rank();
    const int cid = blockIdx.x / cs;
    const int n_clusters = gridDim.x / cs;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nslot = a.nslot;
    const Layout Ly = make_layout(D, G, nslot, a.kpc_max, cs, a.ring_extra, PRE);

    unsigned char *ring = smem + Ly.ring;
    float *coef_t = reinterpret_cast<float *>(smem + Ly.coef_t);
    float *coef_w = reinterpret_cast<float *>(smem + Ly.coef_w);
    double2 *phase = reinterpret_cast<double2 *>(smem + Ly.phase);
    unsigned *whist = reinterpret_cast<unsigned *>(smem + Ly.whist);
    unsigned *bhist = reinterpret_cast<unsigned *>(smem + Ly.bhist);
    int *gh = reinterpret_cast<int *>(smem + Ly.ghist);
    unsigned *lmask = reinterpret_cast<unsigned *>(smem + Ly.lmask);
    unsigned *gmask = reinterpret_cast<unsigned *>(smem + Ly.gmask);
    int *gpre = reinterpret_cast<int *>(smem + Ly.gpre);
    Xch *xch = reinterpret_cast<Xch *>(smem + Ly.xch);
    int *iscratch = reinterpret_cast<int *>(smem + Ly.misc + (kWarps + 1) * 8);
    int *srcidx = reinterpret_cast<int *>(smem + Ly.srcidx);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Ly.bars);

    __shared__ double part_d[kMaxCluster][8], part_q[kMaxCluster][8];
    __shared__ double w_s[kWarps][8], w_q[kWarps][8];
    __shared__ float w_lo[kWarps][8], w_hi[kWarps][8];
    __shared__ float part_lo[kMaxCluster][8], part_hi[kMaxCluster][8];
    __shared__ int part_fail[kMaxCluster];
    __shared__ float muf_s[8], inv_s[8];
    __shared__ int anyfail_s, sel_s[3];

    // this cluster's scratch slot: scores [cap_u][G], then order keys [cap_u]
    float *sc = a.scratch + (long long)cid * a.slot_floats;
    unsigned *ukey = reinterpret_cast<unsigned *>(sc + (long long)a.cap_u * G);
    // (the key stream's evict-first policy is created where a copy is issued: one lane per warp
    // uses it, and a 64-bit register held by every lane would crowd the scoring loop)
    const uint64_t pol_last = policy_evict_last();

    // per-warp TMA buffers; the counters run on across units so that slot and phase
    // parity stay in step with the barriers
    if (lane == 0) {
        for (int k = 0; k < nslot; ++k) mbar_init(bars + warp * nslot + k, 1);
        mbar_init_fence();
    }
    __syncwarp();
    // ring bookkeeping, advanced incrementally (no division by the runtime slot count):
    // the producer fills slot wr_slot; the consumer waits on slot rd_slot for phase rd_phase
    int wr_slot = 0, rd_slot = 0;
    unsigned rd_phase = 0;

    // lane geometry (fixed for the whole launch)
    const int sub = lane % LPK;
    const int kw = lane / LPK;
    int hx = 0;
    {
        int cnt = G;
#pragma unroll
        for (int m = LPK / 2; m >= 1; m >>= 1) {
            if (cnt > 1) {
                const int half = cnt / 2;
                if (lane & m) hx |= half;
                cnt = half;
            }
        }
    }
    const bool writer = (sub & (LPK / G - 1)) == 0;
    const int Hq = a.n_kv * G;

    const int tries = a.wait_tries;  // the drain after a timed-out wait
    // Staggered start. With n_units = q n_clusters + r (0 < r), an even split leaves clusters
    // r.. one unit short, idle at the end; they start about half a unit period late instead.
    // The grid's clusters then no longer reach the memory-bound phases (key stream, compaction)
    // and the latency-bound ones (z-score, select, mask) all at the same time. The period is
    // estimated from unit cid: its algorithmic bytes over the grid's share of 4.6 TB/s.
    if (a.stagger && a.mode == kModePrune && !PRE)
        stagger_wait(a.n_units, n_clusters, cid, a.lens, a.n_kv, a.batch, a.cap_u, a.budget, D);
    // Launched as a programmatic dependent of the validation kernel: everything above overlaps
    // it; the verdicts, the status word and the cache are read only after its completion.
    // (Without a preceding primary grid this returns at once.)
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // Dynamic unit assignment. The kernel launched just before (the validation kernel, or the
    // tensor-core scoring kernel before the precomputed-scores variant) zeroes the counter a.unit_next.
    // Rank 0 takes the cluster's next unit from it just before the unit's moments barrier (where
    // the atomic's latency hides in the wait), and every CTA reads it at the end of the unit; a
    // unit without that barrier takes the next one before an extra barrier. A cluster that
    // started late (placed after other grids' blocks left) or runs slow simply takes fewer units,
    // and ragged units balance over the clusters. The slot of `next`
    // written in iteration it + 1 was last read at the end of iteration it - 1, before that CTA
    // arrived at iteration it's barrier, so no value is overwritten before both CTAs read it.
    auto needs_work = [&](int u) {
        const int su = (u / a.n_kv) % a.batch;
        const int Nu = __ldg(a.lens + su);
        const bool badu = __ldg(a.seq_bad + su) != 0 || Nu < 0 || Nu > a.cap_u;
        return !badu && Nu > 0 && (a.mode == kModeScore || Nu > a.budget);
    };
    // The loop carries nothing in registers (the unit, the iteration count and the cluster's
    // failure flag live in shared memory): a register carried across the whole unit loop spills
    // in the scoring loop, which runs at the register limit.
    __shared__ int unit_s, it_s, dead_s;
    if (tid == 0) {
        it_s = 0;
        dead_s = 0;
    }
    if (crank == 0 && tid == 0) xch->next[0] = (int)atomicAdd(a.unit_next, 1u);
    cluster.sync();
    if (tid == 0) unit_s = ld_rank0_int(&xch->next[0]);
    __syncthreads();
    // the unit after this one, in every thread; two block barriers per unit
    auto advance = [&]() {
        __syncthreads();  // every thread has read this iteration's unit_s and it_s
        if (tid == 0) {
            int nxt = ld_rank0_int(&xch->next[(it_s + 1) & 1]);
            if (dead_s) {
                // the unit already taken is refused like the one whose wait ran out; the
                // cluster takes no more, the other clusters process the rest
                if (nxt < a.n_units && needs_work(nxt) && crank == 0)
                    record_unit_failure(a.status, a.fail_count, a.fail_units, a.fail_cap, kDevTimeout,
                                        a.unit_base + nxt);
                nxt = a.n_units;
            }
            unit_s = nxt;
            ++it_s;
        }
        __syncthreads();
    };
    auto take_next = [&]() {
        if (crank == 0 && tid == 0) xch->next[(it_s + 1) & 1] = (int)atomicAdd(a.unit_next, 1u);
    };
    for (;; advance()) {
        const int unit = unit_s;  // uniform
        if (unit >= a.n_units) break;
        const int g = unit % a.n_kv;
        const int s = (unit / a.n_kv) % a.batch;
        const int lr = unit / (a.n_kv * a.batch);
        const int layer = a.layer_begin + lr;
        const int N = __ldg(a.lens + s);
        // sequences refused by the validation kernel (length, pages, positions against t) are
        // skipped whole; the capacity test is repeated here so that no access depends on it
        const bool bad = __ldg(a.seq_bad + s) != 0 || N < 0 || N > a.cap_u;
        const bool work0 = !bad && N > 0 && (a.mode == kModeScore || N > a.budget);
        bool missing = false;  // the scoring kernel gave up on this unit (it recorded why)
        if constexpr (PRE) missing = work0 && __ldg(a.unit_fail + unit) != 0;
        if (missing && crank == 0 && tid == 0)
            record_unit_failure(a.status, a.fail_count, a.fail_units, a.fail_cap, kDevTimeout, a.unit_base + unit);
        const bool work = work0 && !missing;
        if (!work) {  // uniform over the cluster: no cluster barrier is skipped unevenly
            take_next();  // and the barrier in place of the moments barrier (see above)
            cluster.sync();
            continue;
        }

        const int kpc = ((N + cs - 1) / cs + 31) / 32 * 32;
        const int begin = crank * kpc;
        const int n_local = max(0, min(N - begin, kpc));
        const int nst = (n_local + kStageRows - 1) / kStageRows;
        const int my_stages = warp < nst ? (nst - warp + kWarps - 1) / kWarps : 0;

        float *sc_local = sc + (long long)begin * G;
        const float *sc_read = sc_local;  // where the z pass reads this CTA's scores
        double m_s = 0.0, m_q = 0.0;
        float m_lo = __int_as_float(0x7f800000), m_hi = -__int_as_float(0x7f800000);
        int fail = 0;
        if constexpr (PRE) {
            sc_read = a.pre + ((long long)unit * a.cap_u + begin) * G;
        } else {
        // ---- start streaming this CTA's keys (TMA bulk copies, per-warp buffers) -----
        auto issue = [&](int st, bool withhold) {
            const int slot = wr_slot;
            const int row0 = st * kStageRows;
            const int nrows = min(kStageRows, n_local - row0);
            const long long r = row_of(a, lr, s, g, begin + row0);
            uint64_t *bar = bars + warp * nslot + slot;
            fence_proxy_async_smem();
            mbar_expect_tx(bar, (unsigned)nrows * D * 2u);
            if (withhold) return;
            tma_load_1d(ring + (size_t)(warp * nslot + slot) * kStageBytes, a.K + r * D,
                        (unsigned)nrows * D * 2u, bar, policy_evict_first());
        };
        __syncthreads();  // the ring is free (previous unit's staging reads are done)
        {
            // test hook: the unit's first copy (stage 0: warp 0 of the cluster's first CTA) is
            // withheld, so that the wait for it runs out
            const bool hook = crank == 0 && warp == 0 && a.unit_base + unit == a.inject_unit;
            const int pre = min(nslot, my_stages);
            for (int k = 0; k < pre; ++k) {
                if (lane == 0) issue(warp + k * kWarps, hook && k == 0);
                if (++wr_slot == nslot) wr_slot = 0;
            }
        }

        // ---- prologue: per-head coefficients for this sequence's t --------------------
        const int tq = __ldg(a.t + s);
        for (int f = tid; f < F; f += kThreads) {
            double sn, c;
            sincos(__ldg(a.omega + f) * (double)tq, &sn, &c);
            phase[f] = make_double2(c, sn);
        }
        __syncthreads();
        for (int idx = tid; idx < G * F; idx += kThreads) {
            const int h = idx / F, f = idx % F;
            const long long qi = ((long long)layer * Hq + (long long)g * G + h) * F + f;
            const double2 q = a.Qc[qi];
            const double2 e = phase[f];
            const double re = q.x * e.x - q.y * e.y;
            const double im = q.x * e.y + q.y * e.x;
            const int dre = LAYOUT == 0 ? f : 2 * f;
            const int dim = LAYOUT == 0 ? f + F : 2 * f + 1;
            coef_t[h * D + dre] = (float)re;
            coef_t[h * D + dim] = (float)im;
            coef_w[h * F + f] = __ldg(a.w + qi);
        }
        __syncthreads();

        // register-resident coefficients, in the pair order the unpack produces
        float2 ca[G][NP], cb[G][NP], cw[G][NP];
#pragma unroll
        for (int i = 0; i < G; ++i) {
            const int hq = i ^ hx;
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                const int d0 = pair_dim<LAYOUT>(p, 0), d1 = pair_dim<LAYOUT>(p, 1);
                ca[i][p] = make_float2(coef_t[hq * D + sub * DH + d0], coef_t[hq * D + sub * DH + d1]);
                cb[i][p] = make_float2(coef_t[hq * D + F + sub * DH + d0], coef_t[hq * D + F + sub * DH + d1]);
                int b0;
                if (LAYOUT == 0) {
                    b0 = sub * DH + 2 * p;
                } else {
                    const int base = (p < NP / 2) ? sub * (DH / 2) : D / 4 + sub * (DH / 2);
                    const int q = (p < NP / 2) ? p : p - NP / 2;
                    b0 = base + 2 * q;
                }
                cw[i][p] = make_float2(coef_w[hq * F + b0], coef_w[hq * F + b0 + 1]);
            }
        }

        // ---- score loop ----------------------------------------------------------------
        // writer lanes also gather their head's moments (fp64 sum and sum of squares, fp32
        // min and max) so that the scores are read back only once, for the z-score
        for (int k = 0; k < my_stages; ++k) {
            const int st = warp + k * kWarps;
            const int slot = rd_slot;
            // the key stream's wait keeps the compile-time bound: a runtime bound here costs 3 % of
            // the prune (measured), so the test hook's shorter waits do not apply to it
            const bool landed = __all_sync(FULL, mbar_wait_bounded(bars + warp * nslot + slot, rd_phase, kWaitTries));
            if (!landed) {
                // give the copies this warp still has in flight a bounded chance to land
                int sl = slot;
                unsigned ph = rd_phase;
                for (int j = k + 1; j < min(my_stages, k + nslot); ++j) {
                    if (++sl == nslot) { sl = 0; ph ^= 1u; }
                    (void)mbar_wait_bounded(bars + warp * nslot + sl, ph, tries);
                }
                fail = 1;
                break;
            }
            const uint16_t *stage =
                reinterpret_cast<const uint16_t *>(ring + (size_t)(warp * nslot + slot) * kStageBytes);
            const uint16_t *lane_a = stage + kw * D + sub * DH;
            const int li0 = st * kStageRows + kw;
            float *sc_pass = sc_local + li0 * G + hx;
            const int valid = n_local - li0;  // key of pass p is valid when p * KPP < valid
#pragma unroll
            for (int pass = 0; pass < kStageRows / KPP; ++pass) {
                const uint16_t *row = lane_a + pass * KPP * D;
                unsigned wa[DH / 2], wb[DH / 2];
                load_chunk<DH>(row, wa);
                load_chunk<DH>(row + F, wb);
                float2 xa[NP], xb[NP], nb[NP];
                unpack_pairs<NP, LAYOUT>(wa, xa);
                unpack_pairs<NP, LAYOUT>(wb, xb);
                if (LAYOUT == 0) {
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        const float2 q2 = __ffma2_rn(xb[p], xb[p], __fmul2_rn(xa[p], xa[p]));
                        nb[p] = make_float2(sqrt_approx(q2.x), sqrt_approx(q2.y));
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < NP / 2; ++i) {
                        const float2 qa = __ffma2_rn(xa[2 * i + 1], xa[2 * i + 1], __fmul2_rn(xa[2 * i], xa[2 * i]));
                        const float2 qb = __ffma2_rn(xb[2 * i + 1], xb[2 * i + 1], __fmul2_rn(xb[2 * i], xb[2 * i]));
                        nb[i] = make_float2(sqrt_approx(qa.x), sqrt_approx(qa.y));
                        nb[NP / 2 + i] = make_float2(sqrt_approx(qb.x), sqrt_approx(qb.y));
                    }
                }
                float v[G];
#pragma unroll
                for (int i = 0; i < G; ++i) {
                    float2 acc = __fmul2_rn(xa[0], ca[i][0]);
                    acc = __ffma2_rn(xb[0], cb[i][0], acc);
                    acc = __ffma2_rn(nb[0], cw[i][0], acc);
#pragma unroll
                    for (int p = 1; p < NP; ++p) {
                        acc = __ffma2_rn(xa[p], ca[i][p], acc);
                        acc = __ffma2_rn(xb[p], cb[i][p], acc);
                        acc = __ffma2_rn(nb[p], cw[i][p], acc);
                    }
                    v[i] = acc.x + acc.y;
                }
                // reduce-scatter over the key's LPK lanes: slot i of a lane holds head i ^ hx,
                // so partner lanes always exchange the same register indices.
                {
                    int cnt = G;
#pragma unroll
                    for (int m = LPK / 2; m >= 1; m >>= 1) {
                        if (cnt > 1) {
                            const int half = cnt / 2;
#pragma unroll
                            for (int i = 0; i < half; ++i) v[i] += __shfl_xor_sync(FULL, v[i + half], m);
                            cnt = half;
                        } else {
                            v[0] += __shfl_xor_sync(FULL, v[0], m);
                        }
                    }
                }
                if (writer && pass * KPP < valid) {
                    st_hint(sc_pass + pass * KPP * G, v[0], pol_last);
                    const double dv = (double)v[0];
                    m_s += dv;
                    m_q = fma(dv, dv, m_q);
                    m_lo = fminf(m_lo, v[0]);
                    m_hi = fmaxf(m_hi, v[0]);
                }
            }
            __syncwarp();
            if (++rd_slot == nslot) { rd_slot = 0; rd_phase ^= 1u; }
            if (k + nslot < my_stages) {
                if (lane == 0) issue(warp + (k + nslot) * kWarps, false);
                if (++wr_slot == nslot) wr_slot = 0;
            }
        }
        }  // !PRE
        if (__syncthreads_or(fail)) fail = 1;

        // ---- per-head moments over the whole unit (fp64, cluster-wide) ---------------------
        // Lanes that hold the same head differ only in their key-group bits: fold those in
        // a fixed order, then the warps in order, then the cluster's CTAs in rank order, so
        // that every CTA obtains bit-identical mu and sigma.
        {
            if constexpr (PRE) {
                // every thread folds all G heads of its keys, then the warp folds its lanes
                double ps[G], pq[G];
                float plo[G], phi[G];
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    ps[h] = 0.0;
                    pq[h] = 0.0;
                    plo[h] = __int_as_float(0x7f800000);
                    phi[h] = -__int_as_float(0x7f800000);
                }
                for (int i = tid; i < n_local; i += kThreads) {
                    float sv[G];
                    load_scores<G>(sc_read + (long long)i * G, sv);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const double dv = (double)sv[h];
                        ps[h] += dv;
                        pq[h] = fma(dv, dv, pq[h]);
                        plo[h] = fminf(plo[h], sv[h]);
                        phi[h] = fmaxf(phi[h], sv[h]);
                    }
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        ps[h] += __shfl_xor_sync(FULL, ps[h], o);
                        pq[h] += __shfl_xor_sync(FULL, pq[h], o);
                        plo[h] = fminf(plo[h], __shfl_xor_sync(FULL, plo[h], o));
                        phi[h] = fmaxf(phi[h], __shfl_xor_sync(FULL, phi[h], o));
                    }
                }
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        w_s[warp][h] = ps[h];
                        w_q[warp][h] = pq[h];
                        w_lo[warp][h] = plo[h];
                        w_hi[warp][h] = phi[h];
                    }
                }
            } else {
#pragma unroll
            for (int o = LPK; o < 32; o <<= 1) {
                m_s += __shfl_xor_sync(FULL, m_s, o);
                m_q += __shfl_xor_sync(FULL, m_q, o);
                m_lo = fminf(m_lo, __shfl_xor_sync(FULL, m_lo, o));
                m_hi = fmaxf(m_hi, __shfl_xor_sync(FULL, m_hi, o));
            }
            if (kw == 0 && writer) {
                w_s[warp][hx] = m_s;
                w_q[warp][hx] = m_q;
                w_lo[warp][hx] = m_lo;
                w_hi[warp][hx] = m_hi;
            }
            }
            __syncthreads();
            if (tid < G) {
                double ts_ = 0.0, tq_ = 0.0;
                float lo = __int_as_float(0x7f800000), hi = -lo;
                for (int w = 0; w < kWarps; ++w) {
                    ts_ += w_s[w][tid];
                    tq_ += w_q[w][tid];
                    lo = fminf(lo, w_lo[w][tid]);
                    hi = fmaxf(hi, w_hi[w][tid]);
                }
                xch->sum[tid] = ts_;
                xch->m2[tid] = tq_;
                xch->mn[tid] = lo;
                xch->mx[tid] = hi;
            }
            if (tid == 0) xch->fail = fail;
        }
        take_next();
        cluster.sync();
        // every CTA gathers the cluster's partials (one remote load per thread, all in
        // flight together) and folds them in rank order
        for (int idx = tid; idx < cs * G; idx += kThreads) {
            const int c = idx / G, h = idx % G;
            const Xch *r = cluster.map_shared_rank(xch, c);
            part_d[c][h] = r->sum[h];
            part_q[c][h] = r->m2[h];
            part_lo[c][h] = r->mn[h];
            part_hi[c][h] = r->mx[h];
            if (h == 0) part_fail[c] = r->fail;
        }
        __syncthreads();
        if (tid < G) {
            const int h = tid;
            double tot = 0.0, totq = 0.0;
            float lo = __int_as_float(0x7f800000), hi = -lo;
            for (int c = 0; c < cs; ++c) {
                tot += part_d[c][h];
                totq += part_q[c][h];
                lo = fminf(lo, part_lo[c][h]);
                hi = fmaxf(hi, part_hi[c][h]);
            }
            // population variance from fp64 sums (fp32 scores: no cancellation to fear at
            // fp64 precision); a head whose scores are all equal is flat
            const double mu = tot / (double)N;
            const double var = fmax(totq / (double)N - mu * mu, 0.0);
            const double sigma = sqrt(var);
            const bool flat = !(hi > lo);
            muf_s[h] = (float)mu;
            inv_s[h] = (flat || !(sigma > 0.0)) ? 0.f : (float)(1.0 / sigma);
        }
        if (tid == 32) {
            int f = 0;
            for (int c = 0; c < cs; ++c) f |= part_fail[c];
            anyfail_s = f;
            if (f && crank == 0)
                record_unit_failure(a.status, a.fail_count, a.fail_units, a.fail_cap, kDevTimeout,
                                    a.unit_base + unit);
        }
        __syncthreads();
        if (tid == 0 && anyfail_s) dead_s = 1;  // read after the next block barrier

        // ---- z-score, max over the group, order key --------------------------------------
        // The order keys live in the (now idle) TMA ring when they fit, else in the scratch
        // slot; the first radix digit's histogram is built on the way.
        float *zrow = a.zmax ? a.zmax + (((long long)lr * a.batch + s) * a.n_kv + g) * (long long)a.cap_u + begin
                             : nullptr;
        // raw scores, when asked for, are copied out here from the values read back (the
        // scoring loop stays free of the extra stores)
        float *raw_row = a.raw ? a.raw + (((long long)lr * a.batch + s) * Hq + (long long)g * G) * (long long)a.cap_u + begin
                               : nullptr;
        const bool keys_on_chip = (long long)n_local * 4 <= (long long)Ly.ring_bytes;
        unsigned *uk = keys_on_chip ? reinterpret_cast<unsigned *>(ring) : ukey + begin;
        const bool selecting = a.mode == kModePrune && !anyfail_s;
        {
            unsigned *wh = whist + warp * kBins;
            if (selecting) {
                for (int b = lane; b < kBins; b += 32) wh[b] = 0u;
                __syncwarp();
            }
            float mu_r[G], is_r[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                mu_r[h] = muf_s[h];
                is_r[h] = inv_s[h];
            }
            // the scores come back from L2 in batches: every load of a batch is in flight
            // before the first one is used
            constexpr int ZB = (G >= 8 && LAYOUT == 1) ? 1 : ((G >= 8 || LAYOUT == 1) ? 2 : 4);
            for (int base = tid; base < n_local; base += ZB * kThreads) {
                float sv[ZB][G];
#pragma unroll
                for (int k = 0; k < ZB; ++k) {
                    const int i = base + k * kThreads;
                    if (i < n_local) load_scores<G>(sc_read + (long long)i * G, sv[k]);
                }
                // the next batch is requested into L1 meanwhile (no registers held for it)
#pragma unroll
                for (int k = 0; k < ZB; ++k) {
                    const int i = base + (ZB + k) * kThreads;
                    if (i < n_local) prefetch_l1(sc_read + (long long)i * G);
                }
#pragma unroll
                for (int k = 0; k < ZB; ++k) {
                    const int i = base + k * kThreads;
                    if (i < n_local) {
                        float z = -__int_as_float(0x7f800000);
#pragma unroll
                        for (int h = 0; h < G; ++h) z = fmaxf(z, (sv[k][h] - mu_r[h]) * is_r[h]);
                        z = z + 0.0f;  // -0 -> +0
                        if (zrow) zrow[i] = z;
                        const unsigned key = float_key(z);
                        uk[i] = key;
                        if (selecting) atomicAdd(wh + (key >> 24), 1u);
                    }
                }
            }
            if (raw_row) {
                for (int i = tid; i < n_local; i += kThreads) {
                    float sv[G];
                    load_scores<G>(sc_read + (long long)i * G, sv);
#pragma unroll
                    for (int h = 0; h < G; ++h) raw_row[(long long)h * a.cap_u + i] = sv[h];
                }
            }
        }
        __syncthreads();

        if (selecting) {
            // ---- radix select of the B-th largest key, cluster-wide ------------------------
            unsigned prefix = 0u, pmask = 0u;
            int need = a.budget;
            bool resolved = false;
            for (int pass = 0; pass < 4 && !resolved; ++pass) {
                const int shift = 24 - 8 * pass;
                unsigned *wh = whist + warp * kBins;
                const int lim = pass == 0 ? 0 : n_local;  // pass 0 built above
                if (pass > 0) {
                    for (int b = lane; b < kBins; b += 32) wh[b] = 0u;
                    __syncwarp();
                }
                // the matching keys spread over the bins: plain shared-memory atomics, no
                // warp-level aggregation
                auto count = [&](unsigned u, int i) {
                    if (i < lim && (u & pmask) == prefix) atomicAdd(wh + ((u >> shift) & 255u), 1u);
                };
                if (keys_on_chip) {
                    // four keys per 128-bit load, two loads in flight per thread
                    const uint4 *u4 = reinterpret_cast<const uint4 *>(ring);
                    const int n4 = (lim + 3) / 4;
                    for (int j0 = tid; j0 < n4; j0 += 2 * kThreads) {
                        const int j1 = j0 + kThreads;
                        const uint4 x0 = u4[j0];
                        const uint4 x1 = j1 < n4 ? u4[j1] : make_uint4(0u, 0u, 0u, 0u);
                        count(x0.x, 4 * j0); count(x0.y, 4 * j0 + 1); count(x0.z, 4 * j0 + 2); count(x0.w, 4 * j0 + 3);
                        if (j1 < n4) {
                            count(x1.x, 4 * j1); count(x1.y, 4 * j1 + 1); count(x1.z, 4 * j1 + 2); count(x1.w, 4 * j1 + 3);
                        }
                    }
                } else {
#pragma unroll 4
                    for (int i = tid; i < lim; i += kThreads) count(uk[i], i);
                }
                __syncthreads();
                unsigned *bh = bhist + (pass & 1) * kBins;
                for (int b = tid; b < kBins; b += kThreads) {
                    unsigned c = 0u;
                    for (int w = 0; w < kWarps; ++w) c += whist[w * kBins + b];
                    bh[b] = c;
                }
                cluster.sync();
                // global histogram in top-down order (index 0 = bin 255): thread t folds the
                // cluster's counts of indices [t BPT, t BPT + BPT) in rank order, then a block
                // scan finds the index whose running count first reaches `need` (every CTA
                // folds in the same order and finds the same bin)
                constexpr int BPT = (kBins + kThreads - 1) / kThreads;
                int xs[BPT];
                int tsum = 0;
#pragma unroll
                for (int j = 0; j < BPT; ++j) {
                    const int idx = tid * BPT + j;
                    unsigned c = 0u;
                    if (idx < kBins) {
                        unsigned part[kMaxCluster];
#pragma unroll
                        for (int r = 0; r < kMaxCluster; ++r)
                            part[r] = r < cs ? cluster.map_shared_rank(bh, r)[kBins - 1 - idx] : 0u;
#pragma unroll
                        for (int r = 0; r < kMaxCluster; ++r) c += part[r];
                    }
                    xs[j] = (int)c;
                    tsum += (int)c;
                }
                int incl = tsum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(FULL, incl, o);
                    if (lane >= o) incl += y;
                }
                if (lane == 31) gh[warp] = incl;
                __syncthreads();
                int run = incl - tsum;
                for (int w = 0; w < warp; ++w) run += gh[w];
#pragma unroll
                for (int j = 0; j < BPT; ++j) {
                    const int above = run;
                    run += xs[j];
                    if (above < need && run >= need) {
                        sel_s[0] = kBins - 1 - (tid * BPT + j);
                        sel_s[1] = above;
                        sel_s[2] = xs[j];
                    }
                }
                __syncthreads();
                // gh and sel_s are next written after the next pass's cluster barrier, which
                // every thread reaches only after reading them here: no trailing barrier
                const int bstar = sel_s[0];
                need -= sel_s[1];
                const int cnt = sel_s[2];
                prefix |= (unsigned)bstar << shift;
                pmask |= 255u << shift;
                resolved = (cnt == need);
            }
            const bool tie = !resolved;

            // ---- keep mask: word per 32 local keys; exact ties ranked by slot -------------
            const int nwl = kpc / 32;
            int *tw = gpre;  // scratch for per-word tie counts before gpre is built
            int tie_off = 0;
            if (tie) {
                for (int wi = warp; wi < nwl; wi += kWarps) {
                    const int i = wi * 32 + lane;
                    const bool eq = i < n_local && uk[i] == prefix;
                    const unsigned bb = __ballot_sync(FULL, eq);
                    if (lane == 0) tw[wi] = __popc(bb);
                }
                __syncthreads();
                const int my_ties = block_exclusive_scan<kWarps>(tw, nwl, iscratch);
                if (tid == 0) xch->ties = my_ties;
                cluster.sync();
                if (tid == 0) {
                    int off = 0;
                    for (int c = 0; c < crank; ++c) off += cluster.map_shared_rank(xch, c)->ties;
                    iscratch[kWarps + 1] = off;
                }
                __syncthreads();
                tie_off = iscratch[kWarps + 1];
            }
            // Without ties and with the keys on chip: a lane loads four consecutive keys (one
            // 128-bit load covers 128 keys per warp, i.e. four mask words), forms their keep bits
            // as a nibble, and groups of eight lanes OR their shifted nibbles into one word.
            const int nblk = (nwl + 3) / 4;
            const bool nibble_path = !tie && keys_on_chip && (long long)nblk * 512 <= (long long)Ly.ring_bytes;
            if (nibble_path) {
                const uint4 *u4 = reinterpret_cast<const uint4 *>(ring);
                for (int bk = warp; bk < nblk; bk += kWarps) {
                    const int i0 = bk * 128 + 4 * lane;
                    const uint4 x = u4[bk * 32 + lane];
                    const unsigned uu[4] = {x.x, x.y, x.z, x.w};
                    unsigned nib = 0u;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (i0 + j < n_local && (uu[j] & pmask) >= prefix) nib |= 1u << j;
                    unsigned v = nib << (4 * (lane & 7));
                    v |= __shfl_xor_sync(FULL, v, 1);
                    v |= __shfl_xor_sync(FULL, v, 2);
                    v |= __shfl_xor_sync(FULL, v, 4);
                    const int wi = bk * 4 + (lane >> 3);
                    if ((lane & 7) == 0 && wi < nwl) lmask[wi] = v;
                }
            }
            // otherwise four words per warp per step: their keys are all loaded before the first ballot
            for (int wi0 = warp; wi0 < (nibble_path ? 0 : nwl); wi0 += 4 * kWarps) {
                unsigned uu[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = (wi0 + j * kWarps) * 32 + lane;
                    uu[j] = (wi0 + j * kWarps < nwl && i < n_local) ? uk[i] : 0u;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int wi = wi0 + j * kWarps;
                    if (wi >= nwl) break;  // uniform over the warp
                    const int i = wi * 32 + lane;
                    const bool in = i < n_local;
                    const unsigned u = uu[j];
                    const bool gt = in && (u & pmask) > prefix;
                    const bool eq = in && (u & pmask) == prefix;
                    bool keep = gt || (eq && !tie);
                    if (tie) {
                        const unsigned eb = __ballot_sync(FULL, eq);
                        const int rank = tie_off + tw[wi] + __popc(eb & ((1u << lane) - 1u));
                        keep = gt || (eq && rank < need);
                    }
                    const unsigned kb = __ballot_sync(FULL, keep);
                    if (lane == 0) lmask[wi] = kb;
                }
            }
            cluster.sync();
            // global mask and its word prefix (identical in all CTAs)
            const int nwt = cs * nwl;
            for (int wg = tid; wg < nwt; wg += kThreads) {
                const int c = wg / nwl, wi = wg % nwl;
                const unsigned m = cluster.map_shared_rank(lmask, c)[wi];
                gmask[wg] = m;
                gpre[wg] = __popc(m);
            }
            __syncthreads();
            const int total = block_exclusive_scan<kWarps>(gpre, nwt, iscratch);
            if (tid == 0) gpre[nwt] = total;
            __syncthreads();
            const int M = a.budget;
            // the mask must hold exactly M keys; anything else is an internal error and the
            // unit is left untouched rather than copied from a wrong index
            const bool count_ok = total == M;
            if (!count_ok && crank == 0 && tid == 0)
                record_unit_failure(a.status, a.fail_count, a.fail_units, a.fail_cap, kDevInternal,
                                    a.unit_base + unit);

            // ---- in-place stable compaction ------------------------------------------------
            // Kept rows never move to a higher slot. The only sources a write to [0, M) can
            // clobber are the kept rows below slot M (the first q kept rows, which land in
            // [0, q)). Those move in ascending destination rounds: every CTA first copies its
            // round's sources into shared memory, the cluster synchronises, then all write.
            // The other M - q kept rows come from slots >= M, which no write touches; once the
            // last round's barrier has passed they are copied directly.
            // Two staging buffers in the (idle) TMA ring: the sources of round r + 1 are
            // fetched while round r is written out. Round r + 1 reads slots >= its own
            // destinations, all above the destinations of round r, so the overlap is safe.
            constexpr int LPR = D / 8;  // lanes per row (16 bytes each)
            constexpr int RPW = 32 / LPR;
            const unsigned ring_bytes = Ly.ring_bytes;
            const int S2 = (int)((ring_bytes / 2u) / (unsigned)(4 * D + 4)) / 16 * 16;
            const unsigned buf_bytes = (unsigned)S2 * (4 * D + 4);
            const int wM = M / 32;
            const int q = count_ok ? gpre[wM] + __popc(gmask[wM] & ((1u << (M % 32)) - 1u)) : 0;
            // Paged cache: the sequence's page ids in shared memory (the coefficient area, idle
            // until the next unit), so that a moved row's address needs no global load. The
            // block table row is read once; a table longer than the area keeps the global path.
            const bool pt_smem = a.paged && a.page_shift >= 0 && a.max_pages <= G * D;  // uniform
            const int *pt = reinterpret_cast<const int *>(coef_t);
            if (pt_smem) {
                for (int j = tid; j < a.max_pages; j += kThreads)
                    reinterpret_cast<int *>(coef_t)[j] = __ldg(a.block_table + (long long)s * a.max_pages + j);
                __syncthreads();
            }
            // (the dense check first: the dense path keeps the one test it had)
            auto row_c = [&](int i) -> long long {
                if (!a.paged) return (((long long)lr * a.batch + s) * a.n_kv + g) * (long long)a.cap_u + i;
                if (pt_smem)
                    return (((long long)lr * a.n_pages + pt[i >> a.page_shift]) * a.n_kv + g) * (long long)a.page_size +
                           (i & (a.page_size - 1));
                return row_of(a, lr, s, g, i);
            };
            // source slot of destination dst: the dst-th kept key
            auto source_of = [&](int dst) {
                int lo = 0, hi = nwt;  // largest w with gpre[w] <= dst
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (gpre[mid] <= dst) lo = mid; else hi = mid;
                }
                return min(lo * 32 + select_bit(gmask[lo], dst - gpre[lo]), N - 1);
            };
            const int R = S2 * cs;
            const int H = count_ok ? (q + R - 1) / R : 0;                    // hazard rounds
            const int dfirst = q + crank * S2;
            const int Dk = (count_ok && dfirst < M) ? (M - dfirst + R - 1) / R : 0;  // direct rounds
            const int NR = H + Dk;
            auto round_span = [&](int r, int &nd) {
                int d0;
                if (r < H) {
                    d0 = r * R + crank * S2;
                    nd = max(0, min(q - d0, S2));
                } else {
                    d0 = dfirst + (r - H) * R;
                    nd = max(0, min(M - d0, S2));
                }
                return d0;
            };
            const int qq = lane % LPR;
            auto fetch = [&](int r) {
                int nd;
                const int d0 = round_span(r, nd);
                unsigned char *buf = ring + (r & 1) * buf_bytes;
                uint16_t *stK = reinterpret_cast<uint16_t *>(buf);
                uint16_t *stV = stK + (size_t)S2 * D;
                int32_t *stP = reinterpret_cast<int32_t *>(stV + (size_t)S2 * D);
                int *sidx = srcidx + (r & 1) * S2;
                for (int j = tid; j < nd; j += kThreads) sidx[j] = source_of(d0 + j);
                __syncthreads();
                for (int rr = warp * RPW + lane / LPR; rr < nd; rr += kWarps * RPW) {
                    const long long srow = row_c(sidx[rr]);
                    cp_async16(stK + (size_t)rr * D + qq * 8, a.K + srow * D + qq * 8);
                    cp_async16(stV + (size_t)rr * D + qq * 8, a.V + srow * D + qq * 8);
                    if (qq == 0) cp_async4(stP + rr, a.pos + srow);
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
            };
            if (NR > 0) fetch(0);
            for (int r = 0; r < NR; ++r) {
                if (r + 1 < NR) {
                    fetch(r + 1);
                    asm volatile("cp.async.wait_group 1;" ::: "memory");
                } else {
                    asm volatile("cp.async.wait_group 0;" ::: "memory");
                }
                __syncthreads();
                if (r < H) cluster.sync();  // every source row of this hazard round is on chip
                int nd;
                const int d0 = round_span(r, nd);
                const unsigned char *buf = ring + (r & 1) * buf_bytes;
                const uint16_t *stK = reinterpret_cast<const uint16_t *>(buf);
                const uint16_t *stV = stK + (size_t)S2 * D;
                const int32_t *stP = reinterpret_cast<const int32_t *>(stV + (size_t)S2 * D);
                for (int rr = warp * RPW + lane / LPR; rr < nd; rr += kWarps * RPW) {
                    const long long drow = row_c(d0 + rr);
                    const uint4 xk = *reinterpret_cast<const uint4 *>(stK + (size_t)rr * D + qq * 8);
                    const uint4 xv = *reinterpret_cast<const uint4 *>(stV + (size_t)rr * D + qq * 8);
                    *reinterpret_cast<uint4 *>(a.K + drow * D + qq * 8) = xk;
                    *reinterpret_cast<uint4 *>(a.V + drow * D + qq * 8) = xv;
                    if (qq == 0) a.pos[drow] = stP[rr];
                }
                __syncthreads();
            }
        }
        // No cluster barrier here: the buffers other CTAs read (the exchange record, the
        // histograms, the mask words) are next written after the next unit's moments barrier,
        // which a CTA reaches only after its own reads of this unit's values.
    }
    // a CTA's shared memory must outlive every remote read of it
    cluster.sync();

    // ---- the last CTA to finish publishes the new lengths ------------------------------
    if (a.mode == kModePrune && a.lens_out) {
        __shared__ int last_s;
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            const unsigned tk = atomicAdd(a.counter, 1u);
            last_s = (tk == gridDim.x - 1);
        }
        __syncthreads();
        if (last_s) {
            __threadfence();
            // a sequence refused by the validation kernel keeps its length; every other one
            // gets min(len, B), including one with a unit left uncompacted by a unit-level
            // failure (that unit then holds its first min(len, B) original rows)
            for (int q = tid; q < a.batch; q += kThreads) {
                const int n = a.lens[q];
                a.lens_out[q] = a.seq_bad[q] ? n : min(n, a.budget);
            }
            __syncthreads();
            if (tid == 0) atomicExch(a.counter, 0u);
        }
    }
}

}  // namespace tri
