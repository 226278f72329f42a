// tri_api.cu -- host side of the C ABI declared in include/tri.h.
//
// The statistics loader follows [Deep-dive] §3.4 (offline calibration: load the per-head
// query statistics once) and folds the future-offset average of [Deep-dive] §3.3 into one
// complex constant per band: mean_delta e^{i omega_f (t + delta)} = A_f e^{i omega_f t} with
// A_f = mean_delta e^{i omega_f delta}. Everything that depends on t is formed on the device
// (the phase e^{i omega_f t} in fp64) so that a call never waits on the host.
//
//   [Deep-dive]  "TriAttention深度解析：用三角函数革命性压缩KV Cache，让长推理从「显存地狱」中脱困"
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/tri.h"
#include "tri_kernel.cuh"
#include "tri_calib.cuh"
#include "tri_append.cuh"
#include "tri_maxdelta.cuh"
#include "tri_attend.cuh"

struct tri_ctx {
    int device = -1;
    int sm_count = 0;
    int max_smem_optin = 0;
    // statistics
    bool loaded = false;
    int L = 0, Hkv = 0, G = 0, D = 0, layout = 0;
    double *d_omega = nullptr;
    double2 *d_Qc = nullptr;
    float *d_w = nullptr;
    double2 *d_qbar = nullptr;      // [L][Hq][F] qbar itself (the max-over-offsets mode)
    int64_t *d_offsets = nullptr;   // [n_off]
    int64_t *d_zero_offset = nullptr;  // [1] = {0}: the tensor-core mean mode's single column
    int n_off = 0;
    int combine = TRI_OFFSETS_MEAN;
    int engine = TRI_ENGINE_AUTO;     // which kernels score the mean mode (tri_set_score_engine)
    // scratch of the max-over-offsets mode, grown on demand
    float *d_pre = nullptr;
    size_t pre_bytes = 0;
    unsigned char *d_image = nullptr;
    size_t image_bytes = 0;
    double2 *d_phase = nullptr;
    size_t phase_bytes = 0;
    int32_t *d_tile_prefix = nullptr;
    size_t tile_prefix_bytes = 0;
    int32_t *d_unit_fail = nullptr;
    size_t unit_fail_bytes = 0;
    // chunk partials of tri_decode_attention, grown on demand
    float *d_att_part = nullptr;
    size_t att_part_bytes = 0;
    // device bookkeeping
    unsigned long long *d_status = nullptr;
    // [0] CTAs of the fused kernel done, [1] its next free unit
    unsigned int *d_counter = nullptr;
    int32_t *d_seq_bad = nullptr;    // per-sequence verdict of the validation kernel
    int seq_bad_cap = 0;
    unsigned *d_fail_count = nullptr;  // units left uncompacted by a unit-level failure ...
    int32_t *d_fail_units = nullptr;   // ... the first kFailCap of them
    // test hook (tri_set_test_fault): bounded waits' tries and the unit whose copy is withheld
    int wait_tries = tri::kWaitTries;
    long long inject_unit = -1;
    float *d_scratch = nullptr;      // per-cluster score slots of the persistent grid
    size_t scratch_bytes = 0;
    // tuning (0 = automatic)
    int tune_cs = 0;
    int tune_nslot = 0;
    // text of the last failure seen on the host (CUDA error name and the call that failed)
    char last_error[256] = {0};
    // the last launch shape planned, reused while the call shape and tuning repeat
    struct {
        bool valid = false;
        const void *fn = nullptr;
        long long cap_u = 0, n_units = 0;
        int tune_cs = 0, tune_nslot = 0;
        int cs = 0, nslot = 0, kpc = 0, n_clusters = 0, extra = 0;
        size_t smem = 0;
    } plan_cache;
};

namespace {

// NVTX ranges (domain "tri") around every entry point that launches work, so that a timeline
// profiler shows each call and, in the max-over-offsets mode, each chunk of layers. Without a
// profiler attached a range costs a couple of branches.
nvtxDomainHandle_t nvtx_domain() {
    static nvtxDomainHandle_t d = nvtxDomainCreateA("tri");
    return d;
}

struct NvtxRange {
    explicit NvtxRange(const char *name) {
        nvtxEventAttributes_t e;
        std::memset(&e, 0, sizeof e);
        e.version = NVTX_VERSION;
        e.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
        e.messageType = NVTX_MESSAGE_TYPE_ASCII;
        e.message.ascii = name;
        nvtxDomainRangePushEx(nvtx_domain(), &e);
    }
    ~NvtxRange() { nvtxDomainRangePop(nvtx_domain()); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

using KernelFn = void (*)(const tri::Args);

template <int D, int G, int LAYOUT>
KernelFn kernel_of() {
    return &tri::tri_fused_kernel<D, G, LAYOUT>;
}

KernelFn pick_kernel(int D, int G, int layout) {
#define TRI_CASE(DD, GG)                                                               \
    if (D == DD && G == GG) return layout == 0 ? kernel_of<DD, GG, 0>() : kernel_of<DD, GG, 1>();
    TRI_CASE(64, 1) TRI_CASE(64, 2) TRI_CASE(64, 4) TRI_CASE(64, 8)
    TRI_CASE(128, 1) TRI_CASE(128, 2) TRI_CASE(128, 4) TRI_CASE(128, 8)
#undef TRI_CASE
    return nullptr;
}

bool finite_all(const float *p, size_t n) {
    for (size_t i = 0; i < n; ++i)
        if (!std::isfinite(p[i])) return false;
    return true;
}

void free_stats(tri_ctx *c) {
    cudaFree(c->d_omega);
    cudaFree(c->d_Qc);
    cudaFree(c->d_w);
    cudaFree(c->d_qbar);
    cudaFree(c->d_offsets);
    cudaFree(c->d_zero_offset);
    c->d_zero_offset = nullptr;
    c->d_omega = nullptr;
    c->d_Qc = nullptr;
    c->d_w = nullptr;
    c->d_qbar = nullptr;
    c->d_offsets = nullptr;
    c->n_off = 0;
    c->loaded = false;
}

// The fused kernel reading precomputed scores (the rotary layout plays no part there).
KernelFn pick_pre_kernel(int D, int G) {
#define TRI_CASE(DD, GG) \
    if (D == DD && G == GG) return &tri::tri_fused_kernel<DD, GG, 0, true>;
    TRI_CASE(64, 1) TRI_CASE(64, 2) TRI_CASE(64, 4) TRI_CASE(64, 8)
    TRI_CASE(128, 1) TRI_CASE(128, 2) TRI_CASE(128, 4) TRI_CASE(128, 8)
#undef TRI_CASE
    return nullptr;
}

using MxImageFn = void (*)(const tri::MxArgs);
using MxScoreFn = void (*)(const CUtensorMap, const tri::MxArgs);

bool pick_mx(int D, int G, int layout, int noffp, MxImageFn *img, MxScoreFn *score) {
#define TRI_MX_CASE(DD, GG, LL)                                                        \
    if (D == DD && G == GG && layout == LL) {                                          \
        *img = &tri::tri_mx_image_kernel<DD, GG, LL>;                                  \
        *score = noffp == 1    ? &tri::tri_mx_score_kernel<DD, GG, LL, 1>              \
                 : noffp == 17 ? &tri::tri_mx_score_kernel<DD, GG, LL, 17>             \
                               : &tri::tri_mx_score_kernel<DD, GG, LL, 32>;            \
        return noffp == 1 || noffp == 17 || noffp == 32;                               \
    }
    TRI_MX_CASE(64, 1, 0) TRI_MX_CASE(64, 2, 0) TRI_MX_CASE(64, 4, 0) TRI_MX_CASE(64, 8, 0)
    TRI_MX_CASE(64, 1, 1) TRI_MX_CASE(64, 2, 1) TRI_MX_CASE(64, 4, 1) TRI_MX_CASE(64, 8, 1)
    TRI_MX_CASE(128, 1, 0) TRI_MX_CASE(128, 2, 0) TRI_MX_CASE(128, 4, 0) TRI_MX_CASE(128, 8, 0)
    TRI_MX_CASE(128, 1, 1) TRI_MX_CASE(128, 2, 1) TRI_MX_CASE(128, 4, 1) TRI_MX_CASE(128, 8, 1)
#undef TRI_MX_CASE
    return false;
}

// Device memory check: a pointer the runtime does not know as device or managed memory
// is rejected before anything is launched.
bool is_device_ptr(const void *p) {
    if (!p) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Remember what failed, clear the runtime's sticky-free error state and map to a status.
tri_status cuda_fail(tri_ctx *c, cudaError_t e, const char *what, tri_status st = TRI_ECUDA) {
    if (c) {
        std::snprintf(c->last_error, sizeof c->last_error, "%s: %s (%s)", what, cudaGetErrorName(e),
                      cudaGetErrorString(e));
    }
    cudaGetLastError();
    return st;
}

struct Plan {
    int cs = 0, nslot = 0, kpc = 0, n_clusters = 0, extra = 0;
    size_t smem = 0;
};

// Capacity of the device list of units that a unit-level failure left uncompacted.
constexpr int kFailCap = 4096;

// Live score slots should stay well inside the 126 MB L2 so that the scores written during
// streaming are read back from L2.
constexpr double kScoreL2Budget = 100.0 * 1024 * 1024;
// Fixed cost of a unit in scored keys per CTA (fit to measured prune times of one Qwen3-8B
// layer, 128 units of 2176 keys, over cluster sizes 1 to 16).
constexpr double kUnitOverheadKeys = 700.0;

std::mutex g_attr_mu;

cudaError_t prepare_kernel(KernelFn fn, int max_optin) {
    // Opting in to the full shared-memory carve-out and to 16-CTA clusters is a property
    // of the kernel function, set once per process.
    static std::vector<KernelFn> done;
    std::lock_guard<std::mutex> lk(g_attr_mu);
    if (std::find(done.begin(), done.end(), fn) != done.end()) return cudaSuccess;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             max_optin - (int)fa.sharedSizeBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    done.push_back(fn);
    return cudaSuccess;
}

// Clusters that can be resident at once for this shape (0 if it cannot launch).
int resident_clusters(tri_ctx *c, KernelFn fn, int cs, size_t smem, bool pre) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)cs);
    cfg.blockDim = dim3((unsigned)tri::cta_threads(c->G, pre));
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, fn, &cfg);
    if (e != cudaSuccess) {
        cuda_fail(c, e, "cudaOccupancyMaxActiveClusters");
        return 0;
    }
    return n;
}

// Pick the launch shape of the persistent grid. A cluster of cs CTAs shares one unit; the
// grid holds as many clusters as can be resident (two CTAs per SM). Among the cluster sizes
// whose live score slots (one per resident cluster) fit the L2 budget and whose per-CTA order
// keys fit in shared memory, cs minimises the
// estimated time waves(cs) * (cap_u / cs + kUnitOverheadKeys): the waves of units over the
// resident clusters times a unit's work per CTA plus its fixed cost (prologue, cluster
// exchanges, radix passes and compaction rounds, in key-equivalents). If none fits the budget,
// the largest cs that can launch.
tri_status plan_launch(tri_ctx *c, KernelFn fn, int cap_u, long long n_units, Plan *out, bool pre) {
    auto &pc = c->plan_cache;
    if (pc.valid && pc.fn == (const void *)fn && pc.cap_u == cap_u && pc.n_units == n_units &&
        pc.tune_cs == c->tune_cs && pc.tune_nslot == c->tune_nslot) {
        out->cs = pc.cs;
        out->nslot = pc.nslot;
        out->kpc = pc.kpc;
        out->n_clusters = pc.n_clusters;
        out->extra = pc.extra;
        out->smem = pc.smem;
        return TRI_OK;
    }
    cudaFuncAttributes fa;
    cudaError_t fe = cudaFuncGetAttributes(&fa, fn);
    if (fe != cudaSuccess) return cuda_fail(c, fe, "cudaFuncGetAttributes");
    const size_t budget = (size_t)c->max_smem_optin - fa.sharedSizeBytes;
    // live bytes of a cluster's scratch slot: the scores (fused engine; the order keys usually
    // stay on chip), or only the order keys when the scores come precomputed
    const double unit_bytes = (double)cap_u * (pre ? 1 : c->G) * 4.0;
    const int threads = tri::cta_threads(c->G, pre);
    Plan best;
    bool best_fits = false;
    double best_cost = 0.0;
    for (int cs = 1; cs <= tri::kMaxCluster; cs *= 2) {
        if (c->tune_cs > 0 && cs != c->tune_cs) continue;
        const long long kpc = ((long long)(cap_u + cs - 1) / cs + 31) / 32 * 32;
        if (kpc * cs / 32 > 16384) continue;  // global keep mask must fit on chip
        // buffers per warp: the deepest ring (3 at most) that still leaves room for two
        // CTAs per SM, else whatever fits one CTA
        int nslot = c->tune_nslot > 0 ? c->tune_nslot : 3;
        tri::Layout Ly = tri::make_layout(c->D, c->G, nslot, (int)kpc, cs, 0, pre);
        int res = 0;
        for (; nslot >= 1; --nslot) {
            Ly = tri::make_layout(c->D, c->G, nslot, (int)kpc, cs, 0, pre);
            if (Ly.total > budget || Ly.stage_rows < 16) {
                if (c->tune_nslot > 0) break;
                continue;
            }
            int per_sm = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, Ly.total) != cudaSuccess) {
                cudaGetLastError();
                per_sm = 0;
            }
            if (c->tune_nslot > 0 || per_sm >= tri::kMinBlocks || nslot == 1) {
                res = per_sm >= 1 ? resident_clusters(c, fn, cs, Ly.total, pre) : 0;
                break;
            }
        }
        if (res < 1 || nslot < 1) continue;
        // shared memory left over at this occupancy goes to the compaction's staging
        int extra = 0;
        for (int e = 64 * 1024; e >= 8 * 1024; e -= 8 * 1024) {
            const tri::Layout Le = tri::make_layout(c->D, c->G, nslot, (int)kpc, cs, e, pre);
            if (Le.total > budget) continue;
            int per_sm_e = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_e, fn, threads, Le.total) !=
                cudaSuccess) {
                cudaGetLastError();
                continue;
            }
            int per_sm0 = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm0, fn, threads, Ly.total) !=
                cudaSuccess) {
                cudaGetLastError();
                break;
            }
            if (per_sm_e >= per_sm0) {
                extra = e;
                Ly = Le;
                break;
            }
        }
        Plan p;
        p.extra = extra;
        p.cs = cs;
        p.nslot = nslot;
        p.kpc = (int)kpc;
        p.smem = Ly.total;
        p.n_clusters = (int)std::min<long long>(n_units, res);
        // the order keys of a CTA's share of a unit should fit in the (idle) ring, so that the
        // radix passes run on chip; and the live score slots within the L2 budget
        const bool keys_on_chip = (double)kpc * 4.0 <= (double)Ly.ring_bytes;
        const bool fits_l2 = (double)p.n_clusters * unit_bytes <= kScoreL2Budget && keys_on_chip;
        const double waves = (double)((n_units + res - 1) / res);
        const double cost = waves * ((double)cap_u / cs + kUnitOverheadKeys);
        if (fits_l2 && (!best_fits || cost < best_cost)) {
            best = p;
            best_fits = true;
            best_cost = cost;
        } else if (!best_fits) {
            best = p;  // nothing fits the budget yet: the largest cluster size that launches
        }
    }
    if (best.cs == 0) return TRI_EUNSUPPORTED;
    *out = best;
    pc.valid = true;
    pc.fn = (const void *)fn;
    pc.cap_u = cap_u;
    pc.n_units = n_units;
    pc.tune_cs = c->tune_cs;
    pc.tune_nslot = c->tune_nslot;
    pc.cs = best.cs;
    pc.nslot = best.nslot;
    pc.kpc = best.kpc;
    pc.n_clusters = best.n_clusters;
    pc.extra = best.extra;
    pc.smem = best.smem;
    return TRI_OK;
}

// Host checks of a scoring call (tri_prune / tri_score); on success *cap_out is the unit capacity.
tri_status check_call(tri_ctx *c, const tri_kv *kv, const int32_t *t, int32_t budget, float *raw, float *zmax,
                      int mode, long long *cap_out) {
    if (!c || !kv || !t) return TRI_EINVAL;
    if (!c->loaded) return TRI_ESTATE;
    if (kv->batch < 1 || kv->n_layers < 1 || kv->layer_begin < 0 || kv->layer_begin + kv->n_layers > c->L)
        return TRI_EINVAL;
    const bool paged = kv->block_table != nullptr;
    long long cap_u;
    if (paged) {
        if (kv->page_size < 16 || kv->page_size % 16 != 0 || kv->max_pages < 1 || kv->n_pages < 1)
            return TRI_EINVAL;
        cap_u = (long long)kv->page_size * kv->max_pages;
    } else {
        if (kv->cap < 1) return TRI_EINVAL;
        cap_u = kv->cap;
    }
    if (cap_u > (1LL << 30)) return TRI_EUNSUPPORTED;
    if (mode == tri::kModePrune) {
        if (budget < 1) return TRI_EINVAL;
        if (!kv->K || !kv->V || !kv->pos || !kv->lens) return TRI_EINVAL;
        if (!aligned(kv->K, 16) || !aligned(kv->V, 16) || !aligned(kv->pos, 4)) return TRI_EINVAL;
        if (!is_device_ptr(kv->K) || !is_device_ptr(kv->V) || !is_device_ptr(kv->pos)) return TRI_EINVAL;
        if (kv->lens_out && (!is_device_ptr(kv->lens_out) || !aligned(kv->lens_out, 4))) return TRI_EINVAL;
    } else {
        if (!kv->K || !kv->lens) return TRI_EINVAL;
        if (!aligned(kv->K, 16) || !is_device_ptr(kv->K)) return TRI_EINVAL;
        if (kv->pos && (!aligned(kv->pos, 4) || !is_device_ptr(kv->pos))) return TRI_EINVAL;
        if (raw && (!aligned(raw, 4) || !is_device_ptr(raw))) return TRI_EINVAL;
        if (zmax && (!aligned(zmax, 4) || !is_device_ptr(zmax))) return TRI_EINVAL;
    }
    if (!is_device_ptr(kv->lens) || !is_device_ptr(t) || !aligned(kv->lens, 4) || !aligned(t, 4))
        return TRI_EINVAL;
    if (paged && (!is_device_ptr(kv->block_table) || !aligned(kv->block_table, 4))) return TRI_EINVAL;

    const long long n_units = (long long)kv->n_layers * kv->batch * c->Hkv;
    if (n_units * tri::kMaxCluster > 0x7fffffffLL) return TRI_EUNSUPPORTED;
    *cap_out = cap_u;
    return TRI_OK;
}

// Grow a per-sequence int32 array of the context to `batch` entries (zeroed).
tri_status ensure_flags(int32_t **p, int *cap, int batch) {
    if (batch <= *cap) return TRI_OK;
    cudaFree(*p);  // synchronises the device: no call still uses the old flags
    *p = nullptr;
    *cap = 0;
    if (cudaMalloc(p, sizeof(int32_t) * batch) != cudaSuccess) return TRI_ENOMEM;
    if (cudaMemset(*p, 0, sizeof(int32_t) * batch) != cudaSuccess) return TRI_ECUDA;
    *cap = batch;
    return TRI_OK;
}

tri_status ensure_seq_bad(tri_ctx *c, int batch) { return ensure_flags(&c->d_seq_bad, &c->seq_bad_cap, batch); }

// Arguments shared by the validation kernel and the fused kernel of one call.
tri::Args base_args(tri_ctx *c, const tri_kv *kv, const int32_t *t, int32_t budget, int mode, long long cap_u,
                    int32_t *seq_bad) {
    const bool paged = kv->block_table != nullptr;
    tri::Args a;
    std::memset(&a, 0, sizeof a);
    a.K = static_cast<uint16_t *>(kv->K);
    a.V = static_cast<uint16_t *>(kv->V);
    a.pos = kv->pos;
    a.lens = kv->lens;
    a.block_table = kv->block_table;
    a.t = t;
    a.batch = kv->batch;
    a.n_kv = c->Hkv;
    a.cap_u = (int)cap_u;
    a.paged = paged ? 1 : 0;
    a.page_size = paged ? kv->page_size : 0;
    a.max_pages = paged ? kv->max_pages : 0;
    a.n_pages = paged ? kv->n_pages : 0;
    a.page_shift = -1;
    if (paged && (kv->page_size & (kv->page_size - 1)) == 0)
        for (int b = 0; (1 << b) <= kv->page_size; ++b)
            if ((1 << b) == kv->page_size) a.page_shift = b;
    a.layer_begin = kv->layer_begin;
    a.budget = mode == tri::kModePrune ? budget : 0x7fffffff;
    a.n_units = (int)((long long)kv->n_layers * kv->batch * c->Hkv);
    a.mode = mode;
    a.status = c->d_status;
    a.counter = c->d_counter;
    a.unit_next = c->d_counter + 1;
    a.seq_bad = seq_bad;
    a.wait_tries = c->wait_tries;
    a.inject_unit = c->inject_unit;
    a.fail_count = c->d_fail_count;
    a.fail_units = c->d_fail_units;
    a.fail_cap = kFailCap;
    return a;
}

// The sequence-level checks of a call (tri::tri_validate_kernel), before any unit is touched:
// seq_bad[s] receives each sequence's verdict. Positions are checked against t when the call
// passes them (tri_score may not).
tri_status launch_validate(tri_ctx *c, const tri_kv *kv, const int32_t *t, int mode, long long cap_u,
                           int32_t *seq_bad, void *stream) {
    const tri::Args a = base_args(c, kv, t, 0, mode, cap_u, seq_bad);
    tri::tri_validate_kernel<<<(unsigned)kv->batch, tri::kValidateThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
    const cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess) return cuda_fail(c, ce, "launch(validate)");
    return TRI_OK;
}

// One launch of the fused kernel `fn` over the units of kv. pre / unit_fail: precomputed
// scores (the PRE variant) or null; lens_out: where the last CTA publishes the new lengths
// (null: not in this launch); seq_bad: the validation kernel's per-sequence verdicts.
struct PreScores {  // what the tensor-core scoring kernel left for the fused kernel
    const float *scores = nullptr;
    const int32_t *unit_fail = nullptr;
};

tri_status launch_fused(tri_ctx *c, KernelFn fn, const tri_kv *kv, const int32_t *t, int32_t budget, float *raw,
                        float *zmax, int mode, long long cap_u, const PreScores &pre, long long unit_base,
                        int32_t *lens_out, int32_t *seq_bad, void *stream) {
    const long long n_units = (long long)kv->n_layers * kv->batch * c->Hkv;
    cudaError_t ce = cudaSetDevice(c->device);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaSetDevice");
    ce = prepare_kernel(fn, c->max_smem_optin);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaFuncSetAttribute");
    const bool is_pre = pre.scores != nullptr;
    Plan plan;
    tri_status st = plan_launch(c, fn, (int)cap_u, n_units, &plan, is_pre);
    if (st != TRI_OK) return st;

    const long long slot_floats = ((long long)cap_u * (c->G + 1) + 31) / 32 * 32;
    const size_t need = (size_t)slot_floats * 4 * plan.n_clusters;
    if (need > c->scratch_bytes) {
        cudaFree(c->d_scratch);  // synchronises the device: no call still uses the old slots
        c->d_scratch = nullptr;
        c->scratch_bytes = 0;
        ce = cudaMalloc(&c->d_scratch, need);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaMalloc(scratch)", TRI_ENOMEM);
        c->scratch_bytes = need;
    }

    tri::Args a = base_args(c, kv, t, budget, mode, cap_u, seq_bad);
    a.lens_out = mode == tri::kModePrune ? lens_out : nullptr;
    a.omega = c->d_omega;
    a.Qc = c->d_Qc;
    a.w = c->d_w;
    a.raw = raw;
    a.zmax = zmax;
    a.cs = plan.cs;
    a.kpc_max = plan.kpc;
    a.nslot = plan.nslot;
    a.ring_extra = plan.extra;
    a.scratch = c->d_scratch;
    a.slot_floats = slot_floats;
    a.pre = pre.scores;
    a.unit_fail = pre.unit_fail;
    a.unit_base = unit_base;
    a.stagger = 1;
    // units are handed out from a.unit_next (set by base_args), which the kernel launched just
    // before zeroes: the validation kernel, or the tensor-core scoring kernel of this chunk

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)(plan.n_clusters * plan.cs));
    cfg.blockDim = dim3((unsigned)tri::cta_threads(c->G, is_pre));
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)plan.cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // a programmatic dependent of the validation kernel launched just before on this stream
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    ce = cudaLaunchKernelEx(&cfg, fn, a);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaLaunchKernelEx");
    return TRI_OK;
}

// Grow a scratch buffer of the context (cudaFree synchronises the device, so no call still
// uses the old one).
template <class T>
tri_status grow(tri_ctx *c, T **p, size_t *cap, size_t need, const char *what) {
    if (need <= *cap) return TRI_OK;
    cudaFree(*p);
    *p = nullptr;
    *cap = 0;
    void *q = nullptr;
    const cudaError_t ce = cudaMalloc(&q, need);
    if (ce != cudaSuccess) return cuda_fail(c, ce, what, TRI_ENOMEM);
    *p = static_cast<T *>(q);
    *cap = need;
    return TRI_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// Scores held for at most this many bytes at a time; longer calls run in chunks of layers.
constexpr size_t kMaxPreBytes = size_t(1) << 30;

// The tensor-core engine: per chunk of layers, the tcgen05 scoring kernel writes every unit's
// scores, then the fused kernel's PRE variant z-scores, selects and compacts. With the offsets
// combined by the maximum every (head, offset) is a column; for the mean (mean_tc) a head has
// one column whose coefficient carries the folded offset average, qbar A_f e^{i omega_f t}.
tri_status run_max(tri_ctx *c, const tri_kv *kv, const int32_t *t, int32_t budget, float *raw, float *zmax,
                   int mode, long long cap_u, void *stream, bool mean_tc = false) {
    const int D = c->D, G = c->G, F = D / 2, Hkv = c->Hkv, Hq = Hkv * G;
    const int noffp = mean_tc ? 1 : tri::mx_noff_pad(c->n_off);
    if ((!mean_tc && c->n_off > 32) || G * noffp > 256) {
        std::snprintf(c->last_error, sizeof c->last_error,
                      "max over offsets: %d offsets (padded to %d) for a group of %d exceed the 256 columns of one "
                      "MMA (at most 32 offsets)", c->n_off, noffp, G);
        return TRI_EUNSUPPORTED;
    }
    MxImageFn img_fn = nullptr;
    MxScoreFn score_fn = nullptr;
    if (!pick_mx(D, G, c->layout, noffp, &img_fn, &score_fn)) return TRI_EUNSUPPORTED;
    KernelFn fused = pick_pre_kernel(D, G);
    if (!fused) return TRI_EUNSUPPORTED;
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) {
        std::snprintf(c->last_error, sizeof c->last_error, "cuTensorMapEncodeTiled is not available");
        return TRI_ECUDA;
    }
    const bool paged = kv->block_table != nullptr;
    const int ncol = tri::mx_ncol(G, noffp);
    const unsigned img_bytes = tri::mx_image_bytes(D, G, ncol);
    int piece_rows = 64;
    if (paged) {
        piece_rows = kv->page_size % 64 == 0 ? 64 : kv->page_size % 32 == 0 ? 32 : 16;
    }
    cudaError_t ce = cudaSetDevice(c->device);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaSetDevice");
    cudaFuncAttributes fa;
    ce = cudaFuncGetAttributes(&fa, score_fn);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaFuncGetAttributes(score)");
    const size_t smem_budget = (size_t)c->max_smem_optin - fa.sharedSizeBytes;
    int nst = tri::kMxMaxStages;
    while (nst >= 2 && tri::mx_layout(D, G, ncol, nst).total > smem_budget) --nst;
    if (nst < 2) return TRI_EUNSUPPORTED;
    // at least 120 KB, so that one CTA runs per SM and its TMEM allocation never waits
    const size_t smem = std::max<size_t>(tri::mx_layout(D, G, ncol, nst).total, 120 * 1024);
    ce = cudaFuncSetAttribute(score_fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaFuncSetAttribute(score)");

    // layers per chunk: the scores of one chunk stay under kMaxPreBytes
    const long long units_per_layer = (long long)kv->batch * Hkv;
    const size_t pre_per_layer = (size_t)units_per_layer * cap_u * G * sizeof(float);
    const int chunk = (int)std::max<size_t>(1, std::min<size_t>((size_t)kv->n_layers, kMaxPreBytes / pre_per_layer));
    const long long layer_rows = paged ? (long long)kv->n_pages * Hkv * kv->page_size : units_per_layer * cap_u;
    if (layer_rows * chunk >= (1LL << 31)) return TRI_EUNSUPPORTED;  // TMA row coordinates are int32

    tri_status st;
    if ((st = grow(c, &c->d_pre, &c->pre_bytes, pre_per_layer * chunk, "cudaMalloc(scores)")) != TRI_OK) return st;
    if ((st = grow(c, &c->d_image, &c->image_bytes, (size_t)units_per_layer * chunk * img_bytes,
                   "cudaMalloc(coefficients)")) != TRI_OK)
        return st;
    if ((st = grow(c, &c->d_phase, &c->phase_bytes, (size_t)kv->batch * c->n_off * F * sizeof(double2),
                   "cudaMalloc(phases)")) != TRI_OK)
        return st;
    if ((st = grow(c, &c->d_tile_prefix, &c->tile_prefix_bytes, (size_t)(kv->batch + 1) * sizeof(int32_t),
                   "cudaMalloc(tile prefix)")) != TRI_OK)
        return st;
    if ((st = grow(c, &c->d_unit_fail, &c->unit_fail_bytes, (size_t)units_per_layer * chunk * sizeof(int32_t),
                   "cudaMalloc(unit flags)")) != TRI_OK)
        return st;

    const bool finalize = mode == tri::kModePrune && kv->lens_out != nullptr;
    if ((st = ensure_seq_bad(c, kv->batch)) != TRI_OK) return st;
    if ((st = launch_validate(c, kv, t, mode, cap_u, c->d_seq_bad, stream)) != TRI_OK) return st;

    tri::MxArgs m;
    std::memset(&m, 0, sizeof m);
    m.lens = kv->lens;
    m.block_table = kv->block_table;
    m.t = t;
    m.batch = kv->batch;
    m.n_kv = Hkv;
    m.cap_u = (int)cap_u;
    m.paged = paged ? 1 : 0;
    m.page_size = paged ? kv->page_size : 0;
    m.max_pages = paged ? kv->max_pages : 0;
    m.n_pages = paged ? kv->n_pages : 0;
    m.min_len = mode == tri::kModePrune ? budget : 0;
    m.n_off = mean_tc ? 1 : c->n_off;
    m.noffp = noffp;
    m.ncol = ncol;
    m.nst = nst;
    m.piece_rows = piece_rows;
    m.qbar = mean_tc ? c->d_Qc : c->d_qbar;
    m.omega = c->d_omega;
    m.offsets = mean_tc ? c->d_zero_offset : c->d_offsets;
    m.w = c->d_w;
    m.phase = c->d_phase;
    m.image = c->d_image;
    m.tile_prefix = c->d_tile_prefix;
    m.pre = c->d_pre;
    m.unit_fail = c->d_unit_fail;
    m.status = c->d_status;
    m.seq_bad = c->d_seq_bad;
    m.wait_tries = c->wait_tries;
    m.inject_unit = c->inject_unit;
    m.unit_next = c->d_counter + 1;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);

    tri::tri_mx_prefix_kernel<<<1, 32, 0, cs>>>(m);
    const long long n_ph = (long long)kv->batch * m.n_off * F;
    tri::tri_mx_phase_kernel<<<(unsigned)((n_ph + 255) / 256), 256, 0, cs>>>(m, F);
    ce = cudaGetLastError();
    if (ce != cudaSuccess) return cuda_fail(c, ce, "launch(prefix, phase)");

    for (int lr0 = 0; lr0 < kv->n_layers; lr0 += chunk) {
        NvtxRange chunk_range("tri max-over-offsets: chunk of layers");
        const int nl = std::min(chunk, kv->n_layers - lr0);
        const long long row0 = (long long)lr0 * layer_rows;
        tri_kv sub = *kv;
        sub.layer_begin = kv->layer_begin + lr0;
        sub.n_layers = nl;
        sub.K = static_cast<uint16_t *>(kv->K) + row0 * D;
        if (kv->V) sub.V = static_cast<uint16_t *>(kv->V) + row0 * D;
        if (kv->pos) sub.pos = kv->pos + row0;
        float *raw_c = raw ? raw + (long long)lr0 * kv->batch * Hq * cap_u : nullptr;
        float *zmax_c = zmax ? zmax + (long long)lr0 * units_per_layer * cap_u : nullptr;

        CUtensorMap tmap;
        const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)(layer_rows * nl)};
        const cuuint64_t gstride[1] = {(cuuint64_t)D * 2};
        const cuuint32_t box[2] = {64u, (cuuint32_t)piece_rows};
        const cuuint32_t estride[2] = {1u, 1u};
        const CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sub.K, gdim, gstride, box, estride,
                                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS) {
            std::snprintf(c->last_error, sizeof c->last_error, "cuTensorMapEncodeTiled failed (%d)", (int)cr);
            return TRI_ECUDA;
        }
        m.layer_begin = sub.layer_begin;
        m.n_layers = nl;
        m.unit_base = (long long)lr0 * units_per_layer;
        const long long nu = (long long)nl * units_per_layer;
        img_fn<<<(unsigned)nu, 256, 0, cs>>>(m);
        ce = cudaMemsetAsync(c->d_unit_fail, 0, (size_t)nu * sizeof(int32_t), cs);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaMemsetAsync(unit flags)");
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof cfg);
        cfg.gridDim = dim3((unsigned)c->sm_count);
        cfg.blockDim = dim3((unsigned)tri::mx_threads(G, noffp));
        cfg.dynamicSmemBytes = smem;
        cfg.stream = cs;
        ce = cudaLaunchKernelEx(&cfg, score_fn, tmap, m);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaLaunchKernelEx(score)");
        const bool last = lr0 + nl == kv->n_layers;
        PreScores ps;
        ps.scores = c->d_pre;
        ps.unit_fail = c->d_unit_fail;
        st = launch_fused(c, fused, &sub, t, budget, raw_c, zmax_c, mode, cap_u, ps, m.unit_base,
                          (finalize && last) ? kv->lens_out : nullptr, c->d_seq_bad, stream);
        if (st != TRI_OK) return st;
    }
    return TRI_OK;
}

// The mean mode's engine: the fused CUDA-core kernel, or the tensor-core scoring kernel followed
// by the fused kernel's select and compaction. Automatic: tensor cores at group 8, where the
// folded dot products and norm weights of a key (about 13 flop per key byte) exceed what the
// CUDA cores deliver at the HBM rate; the fused kernel below that (one launch, no score traffic).
bool use_tensor_engine(const tri_ctx *c) {
    if (c->engine == TRI_ENGINE_TENSOR) return true;
    if (c->engine == TRI_ENGINE_CUDA_CORES) return false;
    return c->G >= 8;
}

tri_status run(tri_ctx *c, const tri_kv *kv, const int32_t *t, int32_t budget, float *raw, float *zmax,
               int mode, void *stream) {
    long long cap_u = 0;
    tri_status st = check_call(c, kv, t, budget, raw, zmax, mode, &cap_u);
    if (st != TRI_OK) return st;
    if (c->combine == TRI_OFFSETS_MAX) return run_max(c, kv, t, budget, raw, zmax, mode, cap_u, stream);
    if (use_tensor_engine(c)) return run_max(c, kv, t, budget, raw, zmax, mode, cap_u, stream, true);
    KernelFn fn = pick_kernel(c->D, c->G, c->layout);
    if (!fn) return TRI_EUNSUPPORTED;
    const bool finalize = mode == tri::kModePrune && kv->lens_out != nullptr;
    if ((st = ensure_seq_bad(c, kv->batch)) != TRI_OK) return st;
    if ((st = launch_validate(c, kv, t, mode, cap_u, c->d_seq_bad, stream)) != TRI_OK) return st;
    return launch_fused(c, fn, kv, t, budget, raw, zmax, mode, cap_u, PreScores(), 0,
                        finalize ? kv->lens_out : nullptr, c->d_seq_bad, stream);
}

// ---------------------------------------------------------------------------------------
// Allocation-free prune. Some callers cannot allocate device memory at call time: a serving
// loop whose device memory is owned by another allocator, or one that cannot afford the
// device-wide synchronisation that cudaFree implies when tri_prune has to grow its scratch.
// For them the per-cluster score slots (and the per-sequence validation verdicts) live in
// file-scope device arrays of fixed size, loaded with the library and held until exit.
// ---------------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // score slots: 64 MiB
constexpr int kNoAllocMaxBatch = 16384;                       // validation verdicts
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];
static __device__ __align__(256) int32_t g_noalloc_seq_bad[kNoAllocMaxBatch];

struct NoAllocSymbols {
    bool ready = false;
    float *scratch = nullptr;
    int32_t *seq_bad = nullptr;
};
std::mutex g_noalloc_mu;
NoAllocSymbols g_noalloc[kMaxDevices];

// Device addresses of the two arrays on the context's device (set up once per device, with
// that device current). The host-side names are stand-ins, never device addresses.
tri_status noalloc_symbols(tri_ctx *c, NoAllocSymbols *out) {
    if (c->device < 0 || c->device >= kMaxDevices) return TRI_EUNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoAllocSymbols &e = g_noalloc[c->device];
    if (!e.ready) {
        cudaError_t ce = cudaSetDevice(c->device);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaSetDevice");
        void *p = nullptr;
        ce = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaGetSymbolAddress(g_noalloc_scratch)");
        e.scratch = static_cast<float *>(p);
        p = nullptr;
        ce = cudaGetSymbolAddress(&p, g_noalloc_seq_bad);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaGetSymbolAddress(g_noalloc_seq_bad)");
        e.seq_bad = static_cast<int32_t *>(p);
        e.ready = true;
    }
    *out = e;
    return TRI_OK;
}

tri_status run_noalloc(tri_ctx *c, const tri_kv *kv, const int32_t *t, int32_t budget, void *stream) {
    if (!c || !kv || !t) return TRI_EINVAL;
    if (!c->loaded) return TRI_ESTATE;
    if (c->combine != TRI_OFFSETS_MEAN) {
        std::snprintf(c->last_error, sizeof c->last_error,
                      "tri_prune_noalloc: the max-over-offsets mode needs scratch that only tri_prune allocates");
        return TRI_EUNSUPPORTED;
    }
    if (kv->batch < 1 || kv->n_layers < 1 || kv->layer_begin < 0 || kv->layer_begin + kv->n_layers > c->L)
        return TRI_EINVAL;
    const bool paged = kv->block_table != nullptr;
    long long cap_u;
    if (paged) {
        if (kv->page_size < 16 || kv->page_size % 16 != 0 || kv->max_pages < 1 || kv->n_pages < 1)
            return TRI_EINVAL;
        cap_u = (long long)kv->page_size * kv->max_pages;
    } else {
        if (kv->cap < 1) return TRI_EINVAL;
        cap_u = kv->cap;
    }
    if (cap_u > (1LL << 30)) return TRI_EUNSUPPORTED;
    if (budget < 1) return TRI_EINVAL;
    if (!kv->K || !kv->V || !kv->pos || !kv->lens) return TRI_EINVAL;
    if (!aligned(kv->K, 16) || !aligned(kv->V, 16) || !aligned(kv->pos, 4)) return TRI_EINVAL;
    if (!is_device_ptr(kv->K) || !is_device_ptr(kv->V) || !is_device_ptr(kv->pos)) return TRI_EINVAL;
    if (kv->lens_out && (!is_device_ptr(kv->lens_out) || !aligned(kv->lens_out, 4))) return TRI_EINVAL;
    if (!is_device_ptr(kv->lens) || !is_device_ptr(t) || !aligned(kv->lens, 4) || !aligned(t, 4))
        return TRI_EINVAL;
    if (paged && (!is_device_ptr(kv->block_table) || !aligned(kv->block_table, 4))) return TRI_EINVAL;
    if (kv->batch > kNoAllocMaxBatch) {
        std::snprintf(c->last_error, sizeof c->last_error,
                      "tri_prune_noalloc: batch %d exceeds the fixed flag array (%d sequences)", kv->batch,
                      kNoAllocMaxBatch);
        return TRI_EUNSUPPORTED;
    }
    const long long n_units = (long long)kv->n_layers * kv->batch * c->Hkv;
    if (n_units * tri::kMaxCluster > 0x7fffffffLL) return TRI_EUNSUPPORTED;

    KernelFn fn = pick_kernel(c->D, c->G, c->layout);
    if (!fn) return TRI_EUNSUPPORTED;
    cudaError_t ce = cudaSetDevice(c->device);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaSetDevice");
    NoAllocSymbols sym;
    tri_status st = noalloc_symbols(c, &sym);
    if (st != TRI_OK) return st;
    ce = prepare_kernel(fn, c->max_smem_optin);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaFuncSetAttribute");
    Plan plan;
    st = plan_launch(c, fn, (int)cap_u, n_units, &plan, false);
    if (st == TRI_EUNSUPPORTED) {
        std::snprintf(c->last_error, sizeof c->last_error,
                      "tri_prune_noalloc: no launch shape holds a unit capacity of %lld slots on chip", cap_u);
        return st;
    }
    if (st != TRI_OK) return st;

    // as many resident clusters as the fixed scratch holds slots for (the grid is persistent,
    // so fewer clusters still cover every unit)
    const long long slot_floats = ((long long)cap_u * (c->G + 1) + 31) / 32 * 32;
    const long long slots = (long long)(kNoAllocScratchBytes / sizeof(float)) / slot_floats;
    if (slots < 1) {
        std::snprintf(c->last_error, sizeof c->last_error,
                      "tri_prune_noalloc: a unit of %lld slots needs %lld bytes of scratch, above the fixed "
                      "%zu bytes (at most %lld slots per unit for this group size)",
                      cap_u, slot_floats * 4, kNoAllocScratchBytes,
                      (long long)(kNoAllocScratchBytes / sizeof(float)) / (c->G + 1) / 32 * 32);
        return TRI_EUNSUPPORTED;
    }
    const int n_clusters = (int)std::min<long long>(plan.n_clusters, slots);

    // the per-sequence verdicts go to the fixed flag array, written whole by the validation kernel
    st = launch_validate(c, kv, t, tri::kModePrune, cap_u, sym.seq_bad, stream);
    if (st != TRI_OK) return st;

    tri::Args a = base_args(c, kv, t, budget, tri::kModePrune, cap_u, sym.seq_bad);
    a.lens_out = kv->lens_out;
    a.omega = c->d_omega;
    a.Qc = c->d_Qc;
    a.w = c->d_w;
    a.cs = plan.cs;
    a.kpc_max = plan.kpc;
    a.nslot = plan.nslot;
    a.ring_extra = plan.extra;
    a.scratch = sym.scratch;
    a.slot_floats = slot_floats;
    a.stagger = 1;

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)(n_clusters * plan.cs));
    cfg.blockDim = dim3((unsigned)tri::cta_threads(c->G));
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)plan.cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // a programmatic dependent of the validation kernel launched just before on this stream
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    ce = cudaLaunchKernelEx(&cfg, fn, a);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaLaunchKernelEx");
    return TRI_OK;
}

using CalPartialFn = void (*)(const uint16_t *, int, int, int, double *);
using CalFinalFn = void (*)(const double *, int, int, int, int, float *, float *, float *);

bool pick_calib(int D, int layout, CalPartialFn *p, CalFinalFn *f) {
#define TRI_CAL_CASE(DD, LL)                                    \
    if (D == DD && layout == LL) {                              \
        *p = &tri::tri_calib_partial_kernel<DD, LL>;            \
        *f = &tri::tri_calib_final_kernel<DD, LL>;              \
        return true;                                            \
    }
    TRI_CAL_CASE(64, 0) TRI_CAL_CASE(64, 1) TRI_CAL_CASE(128, 0) TRI_CAL_CASE(128, 1)
#undef TRI_CAL_CASE
    return false;
}

using AttFn = void (*)(const tri::AttArgs);

bool pick_attend(int D, int G, AttFn *main_fn, AttFn *combine_fn) {
#define TRI_ATT_CASE(DD, GG)                                      \
    if (D == DD && G == GG) {                                     \
        *main_fn = &tri::tri_attend_kernel<DD, GG>;               \
        *combine_fn = &tri::tri_attend_combine_kernel<DD, GG>;    \
        return true;                                              \
    }
    TRI_ATT_CASE(64, 1) TRI_ATT_CASE(64, 2) TRI_ATT_CASE(64, 4) TRI_ATT_CASE(64, 8)
    TRI_ATT_CASE(128, 1) TRI_ATT_CASE(128, 2) TRI_ATT_CASE(128, 4) TRI_ATT_CASE(128, 8)
#undef TRI_ATT_CASE
    return false;
}

tri_status run_attend(tri_ctx *c, const tri_kv *kv, const void *q, float *out, void *stream) {
    if (!c || !kv || !q || !out) return TRI_EINVAL;
    if (!c->loaded) return TRI_ESTATE;
    if (kv->batch < 1 || kv->n_layers < 1 || kv->layer_begin < 0 || kv->layer_begin + kv->n_layers > c->L)
        return TRI_EINVAL;
    const bool paged = kv->block_table != nullptr;
    long long cap_u;
    if (paged) {
        if (kv->page_size < 16 || kv->page_size % 16 != 0 || kv->max_pages < 1 || kv->n_pages < 1)
            return TRI_EINVAL;
        cap_u = (long long)kv->page_size * kv->max_pages;
    } else {
        if (kv->cap < 1) return TRI_EINVAL;
        cap_u = kv->cap;
    }
    if (cap_u > (1LL << 30)) return TRI_EUNSUPPORTED;
    if (!kv->K || !kv->V || !kv->lens) return TRI_EINVAL;
    if (!aligned(kv->K, 16) || !aligned(kv->V, 16) || !aligned(q, 16) || !aligned(out, 4) ||
        !aligned(kv->lens, 4))
        return TRI_EINVAL;
    if (!is_device_ptr(kv->K) || !is_device_ptr(kv->V) || !is_device_ptr(q) || !is_device_ptr(out) ||
        !is_device_ptr(kv->lens))
        return TRI_EINVAL;
    if (paged && (!is_device_ptr(kv->block_table) || !aligned(kv->block_table, 4))) return TRI_EINVAL;
    AttFn fn = nullptr, comb = nullptr;
    if (!pick_attend(c->D, c->G, &fn, &comb)) return TRI_EUNSUPPORTED;
    const long long n_units = (long long)kv->n_layers * kv->batch * c->Hkv;
    if (n_units > 0x7fffffffLL) return TRI_EUNSUPPORTED;
    cudaError_t ce = cudaSetDevice(c->device);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaSetDevice");

    // launch shape: the deepest per-warp ring (3 stages at most) that keeps three CTAs per SM,
    // else the ring depth that gives the most CTAs per SM (registers may allow only two)
    ce = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)tri::att_smem_bytes(c->D, c->G, 3));
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaFuncSetAttribute(attend)");
    int nslot = 0, per_sm = 0;
    for (int ns = 3; ns >= 1; --ns) {
        int p = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&p, fn, tri::kAttThreads,
                                                          tri::att_smem_bytes(c->D, c->G, ns)) != cudaSuccess) {
            cudaGetLastError();
            continue;
        }
        if (p > per_sm) {
            per_sm = p;
            nslot = ns;
        }
        if (p >= 3) break;
    }
    if (per_sm < 1 || nslot < 1) return TRI_EUNSUPPORTED;
    // chunks per unit: split the units' rows only when there are too few units for four waves
    const long long target = 4LL * c->sm_count * per_sm;
    long long cpu = (target + n_units - 1) / n_units;
    cpu = std::max<long long>(1, std::min<long long>(cpu, (cap_u + 255) / 256));
    if (n_units * cpu > 0x7fffffffLL) return TRI_EUNSUPPORTED;

    tri_status st = ensure_seq_bad(c, kv->batch);
    if (st != TRI_OK) return st;
    if (cpu > 1) {
        const size_t need = (size_t)n_units * cpu * c->G * (c->D + 2) * sizeof(float);
        if ((st = grow(c, &c->d_att_part, &c->att_part_bytes, need, "cudaMalloc(attention partials)")) != TRI_OK)
            return st;
    }
    // sequence-level checks (length, pages; no positions: the attention does not read them)
    tri_kv chk = *kv;
    chk.pos = nullptr;
    if ((st = launch_validate(c, &chk, nullptr, tri::kModeScore, cap_u, c->d_seq_bad, stream)) != TRI_OK) return st;

    tri::AttArgs a;
    std::memset(&a, 0, sizeof a);
    a.K = static_cast<const uint16_t *>(kv->K);
    a.V = static_cast<const uint16_t *>(kv->V);
    a.q = static_cast<const uint16_t *>(q);
    a.out = out;
    a.part = c->d_att_part;
    a.lens = kv->lens;
    a.block_table = kv->block_table;
    a.seq_bad = c->d_seq_bad;
    a.batch = kv->batch;
    a.n_kv = c->Hkv;
    a.cap_u = (int)cap_u;
    a.paged = paged ? 1 : 0;
    a.page_size = paged ? kv->page_size : 0;
    a.max_pages = paged ? kv->max_pages : 0;
    a.n_pages = paged ? kv->n_pages : 0;
    a.n_units = (int)n_units;
    a.cpu = (int)cpu;
    a.nslot = nslot;
    a.qscale = (float)(1.4426950408889634 / std::sqrt((double)c->D));
    a.status = c->d_status;
    a.wait_tries = c->wait_tries;
    // each launch a programmatic dependent of the one before on this stream (the validation, then
    // the attention): its launch overlaps the previous grid's end; the kernels wait before they
    // read what it wrote
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)(n_units * cpu));
    cfg.blockDim = dim3((unsigned)tri::kAttThreads);
    cfg.dynamicSmemBytes = tri::att_smem_bytes(c->D, c->G, nslot);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    ce = cudaLaunchKernelEx(&cfg, fn, a);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "launch(attend)");
    if (cpu > 1) {
        cfg.gridDim = dim3((unsigned)n_units);
        cfg.blockDim = dim3(256u);
        cfg.dynamicSmemBytes = 0;
        ce = cudaLaunchKernelEx(&cfg, comb, a);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "launch(attend combine)");
    }
    return TRI_OK;
}

}  // namespace

extern "C" {

tri_status tri_create(tri_ctx **out, int device) {
    if (!out) return TRI_EINVAL;
    *out = nullptr;
    int n = 0;
    if (cudaGetDeviceCount(&n) != cudaSuccess) {
        cudaGetLastError();
        return TRI_ECUDA;
    }
    if (device < 0 || device >= n) return TRI_EINVAL;
    cudaDeviceProp p;
    if (cudaGetDeviceProperties(&p, device) != cudaSuccess) return TRI_ECUDA;
    if (p.major != 10) return TRI_EUNSUPPORTED;
    if (cudaSetDevice(device) != cudaSuccess) return TRI_ECUDA;
    tri_ctx *c = new (std::nothrow) tri_ctx;
    if (!c) return TRI_ENOMEM;
    c->device = device;
    c->sm_count = p.multiProcessorCount;
    c->max_smem_optin = (int)p.sharedMemPerBlockOptin;
    if (cudaMalloc(&c->d_status, sizeof(unsigned long long)) != cudaSuccess ||
        cudaMalloc(&c->d_counter, 2 * sizeof(unsigned int)) != cudaSuccess ||
        cudaMalloc(&c->d_fail_count, sizeof(unsigned)) != cudaSuccess ||
        cudaMalloc(&c->d_fail_units, sizeof(int32_t) * kFailCap) != cudaSuccess) {
        tri_destroy(c);
        return TRI_ENOMEM;
    }
    if (cudaMemset(c->d_status, 0, sizeof(unsigned long long)) != cudaSuccess ||
        cudaMemset(c->d_counter, 0, 2 * sizeof(unsigned int)) != cudaSuccess ||
        cudaMemset(c->d_fail_count, 0, sizeof(unsigned)) != cudaSuccess) {
        tri_destroy(c);
        return TRI_ECUDA;
    }
    *out = c;
    return TRI_OK;
}

tri_status tri_destroy(tri_ctx *c) {
    if (!c) return TRI_OK;
    if (c->device >= 0) cudaSetDevice(c->device);
    free_stats(c);
    cudaFree(c->d_status);
    cudaFree(c->d_counter);
    cudaFree(c->d_seq_bad);
    cudaFree(c->d_fail_count);
    cudaFree(c->d_fail_units);
    cudaFree(c->d_scratch);
    cudaFree(c->d_pre);
    cudaFree(c->d_image);
    cudaFree(c->d_phase);
    cudaFree(c->d_tile_prefix);
    cudaFree(c->d_unit_fail);
    cudaFree(c->d_att_part);
    delete c;
    return TRI_OK;
}

tri_status tri_calibrate_load(tri_ctx *c, int n_layers, int n_kv_heads, int group, int head_dim,
                              double rope_base, tri_rope_layout layout, const float *q_mean,
                              const float *q_norm_mean, const float *R, const int64_t *offsets,
                              int n_offsets) {
    if (!c) return TRI_EINVAL;
    if (n_layers < 1 || n_kv_heads < 1 || n_offsets < 1) return TRI_EINVAL;
    if (head_dim != 64 && head_dim != 128) return TRI_EINVAL;
    if (group != 1 && group != 2 && group != 4 && group != 8) return TRI_EINVAL;
    if (!(rope_base > 0.0) || !std::isfinite(rope_base)) return TRI_EINVAL;
    if (layout != TRI_ROPE_HALF && layout != TRI_ROPE_INTERLEAVED) return TRI_EINVAL;
    if (!q_mean || !q_norm_mean || !R || !offsets) return TRI_EINVAL;
    const int D = head_dim, F = D / 2, Hq = n_kv_heads * group;
    const size_t nq = (size_t)n_layers * Hq * D, nb = (size_t)n_layers * Hq * F;
    if (!finite_all(q_mean, nq) || !finite_all(q_norm_mean, nb) || !finite_all(R, nb)) return TRI_EINVAL;

    // fp64 constants: omega_f = base^(-2f/d) and the offset average A_f
    std::vector<double> omega(F);
    std::vector<double> Are(F), Aim(F);
    for (int f = 0; f < F; ++f) {
        omega[f] = std::pow(rope_base, -2.0 * (double)f / (double)D);
        double sr = 0.0, si = 0.0;
        for (int j = 0; j < n_offsets; ++j) {
            const double ang = omega[f] * (double)offsets[j];
            sr += std::cos(ang);
            si += std::sin(ang);
        }
        Are[f] = sr / n_offsets;
        Aim[f] = si / n_offsets;
    }
    std::vector<double2> Qc(nb), qbar(nb);
    std::vector<float> w(nb);
    for (size_t lh = 0; lh < (size_t)n_layers * Hq; ++lh) {
        const float *q = q_mean + lh * D;
        for (int f = 0; f < F; ++f) {
            const int dre = layout == TRI_ROPE_HALF ? f : 2 * f;
            const int dim = layout == TRI_ROPE_HALF ? f + F : 2 * f + 1;
            const double qr = q[dre], qi = q[dim];
            Qc[lh * F + f] = make_double2(qr * Are[f] - qi * Aim[f], qr * Aim[f] + qi * Are[f]);
            qbar[lh * F + f] = make_double2(qr, qi);
            w[lh * F + f] = (float)((1.0 - (double)R[lh * F + f]) * (double)q_norm_mean[lh * F + f]);
        }
    }
    if (cudaSetDevice(c->device) != cudaSuccess) return TRI_ECUDA;
    free_stats(c);
    if (cudaMalloc(&c->d_omega, sizeof(double) * F) != cudaSuccess ||
        cudaMalloc(&c->d_Qc, sizeof(double2) * nb) != cudaSuccess ||
        cudaMalloc(&c->d_w, sizeof(float) * nb) != cudaSuccess ||
        cudaMalloc(&c->d_qbar, sizeof(double2) * nb) != cudaSuccess ||
        cudaMalloc(&c->d_offsets, sizeof(int64_t) * n_offsets) != cudaSuccess ||
        cudaMalloc(&c->d_zero_offset, sizeof(int64_t)) != cudaSuccess) {
        free_stats(c);
        return TRI_ENOMEM;
    }
    if (cudaMemcpy(c->d_omega, omega.data(), sizeof(double) * F, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->d_Qc, Qc.data(), sizeof(double2) * nb, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->d_w, w.data(), sizeof(float) * nb, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->d_qbar, qbar.data(), sizeof(double2) * nb, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(c->d_offsets, offsets, sizeof(int64_t) * n_offsets, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemset(c->d_zero_offset, 0, sizeof(int64_t)) != cudaSuccess) {
        free_stats(c);
        return TRI_ECUDA;
    }
    c->n_off = n_offsets;
    c->L = n_layers;
    c->Hkv = n_kv_heads;
    c->G = group;
    c->D = D;
    c->layout = layout;
    c->loaded = true;
    return TRI_OK;
}

tri_status tri_prune(tri_ctx *c, const tri_kv *kv, const int32_t *t, int32_t budget, void *stream) {
    NvtxRange r("tri_prune");
    return run(c, kv, t, budget, nullptr, nullptr, tri::kModePrune, stream);
}

tri_status tri_prune_noalloc(tri_ctx *c, const tri_kv *kv, const int32_t *t, int32_t budget, void *stream) {
    NvtxRange r("tri_prune_noalloc");
    return run_noalloc(c, kv, t, budget, stream);
}

tri_status tri_score(tri_ctx *c, const tri_kv *kv, const int32_t *t, float *raw, float *zmax, void *stream) {
    NvtxRange r("tri_score");
    return run(c, kv, t, 0, raw, zmax, tri::kModeScore, stream);
}

tri_status tri_decode_attention(tri_ctx *c, const tri_kv *kv, const void *q, float *out, void *stream) {
    NvtxRange r("tri_decode_attention");
    return run_attend(c, kv, q, out, stream);
}

tri_status tri_calibrate_estimate(tri_ctx *c, const void *Q, int n_layers, int T, int n_q_heads, int head_dim,
                                  tri_rope_layout layout, float *q_mean, float *q_norm_mean, float *R,
                                  void *stream) {
    NvtxRange r("tri_calibrate_estimate");
    if (!c || !Q || !q_mean || !q_norm_mean || !R) return TRI_EINVAL;
    if (n_layers < 1 || T < 1 || n_q_heads < 1) return TRI_EINVAL;
    if (layout != TRI_ROPE_HALF && layout != TRI_ROPE_INTERLEAVED) return TRI_EINVAL;
    CalPartialFn pk = nullptr;
    CalFinalFn fk = nullptr;
    if (!pick_calib(head_dim, (int)layout, &pk, &fk)) return TRI_EUNSUPPORTED;
    if (!aligned(Q, 16) || !aligned(q_mean, 4) || !aligned(q_norm_mean, 4) || !aligned(R, 4)) return TRI_EINVAL;
    if (!is_device_ptr(Q) || !is_device_ptr(q_mean) || !is_device_ptr(q_norm_mean) || !is_device_ptr(R))
        return TRI_EINVAL;
    const long long n_chunks = ((long long)T + tri::kCalChunk - 1) / tri::kCalChunk;
    const long long bands = (long long)n_layers * n_q_heads * (head_dim / 2);
    const long long cols = (long long)n_q_heads * (head_dim / 2 / tri::kCalBands);
    const long long groups = (cols + tri::kCalThreads - 1) / tri::kCalThreads;
    if (n_layers > 65535 || groups > 65535 || n_chunks > 0x7fffffffLL) return TRI_EUNSUPPORTED;
    cudaError_t ce = cudaSetDevice(c->device);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaSetDevice");
    const size_t need = (size_t)n_chunks * (size_t)bands * 3 * sizeof(double);
    if (need > c->scratch_bytes) {
        cudaFree(c->d_scratch);  // synchronises the device: no call still uses the old scratch
        c->d_scratch = nullptr;
        c->scratch_bytes = 0;
        ce = cudaMalloc(&c->d_scratch, need);
        if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaMalloc(scratch)", TRI_ENOMEM);
        c->scratch_bytes = need;
    }
    double *part = reinterpret_cast<double *>(c->d_scratch);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const dim3 grid1((unsigned)n_chunks, (unsigned)n_layers, (unsigned)groups);
    pk<<<grid1, tri::kCalThreads, 0, st>>>(static_cast<const uint16_t *>(Q), n_layers, T, n_q_heads, part);
    ce = cudaGetLastError();
    if (ce != cudaSuccess) return cuda_fail(c, ce, "calibration partial sums");
    const dim3 grid2((unsigned)((bands + tri::kCalThreads - 1) / tri::kCalThreads));
    fk<<<grid2, tri::kCalThreads, 0, st>>>(part, (int)n_chunks, n_layers, T, n_q_heads, q_mean, q_norm_mean, R);
    ce = cudaGetLastError();
    if (ce != cudaSuccess) return cuda_fail(c, ce, "calibration means");
    return TRI_OK;
}

namespace {
tri_status append_impl(tri_ctx *c, const tri_kv *kv, const void *K_new, const void *V_new, const int32_t *pos_new,
                       bool advance, void *stream) {
    if (!c || !kv || !K_new || !V_new || !pos_new) return TRI_EINVAL;
    if (!c->loaded) return TRI_ESTATE;
    if (c->D != 64 && c->D != 128) return TRI_EUNSUPPORTED;
    if (!kv->block_table || !kv->K || !kv->V || !kv->pos || !kv->lens || !kv->lens_out) return TRI_EINVAL;
    if (kv->batch < 1 || kv->n_layers < 1 || kv->layer_begin < 0 || kv->layer_begin + kv->n_layers > c->L)
        return TRI_EINVAL;
    if (kv->page_size < 16 || kv->page_size % 16 != 0 || kv->max_pages < 1 || kv->n_pages < 1) return TRI_EINVAL;
    const void *dev[] = {kv->K, kv->V, kv->pos, kv->lens, kv->lens_out, kv->block_table, K_new, V_new, pos_new};
    for (const void *p : dev)
        if (!is_device_ptr(p)) return TRI_EINVAL;
    if (!aligned(kv->K, 16) || !aligned(kv->V, 16) || !aligned(K_new, 16) || !aligned(V_new, 16) ||
        !aligned(kv->pos, 4) || !aligned(kv->lens, 4) || !aligned(kv->lens_out, 4) || !aligned(pos_new, 4) ||
        !aligned(kv->block_table, 4))
        return TRI_EINVAL;
    const int cs = tri::append_cluster_size((long long)kv->n_layers * c->Hkv);
    if ((long long)kv->batch * cs > 0x7fffffffLL) return TRI_EUNSUPPORTED;
    cudaError_t ce = cudaSetDevice(c->device);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "cudaSetDevice");
    tri::AppendArgs a;
    a.K = static_cast<uint16_t *>(kv->K);
    a.V = static_cast<uint16_t *>(kv->V);
    a.pos = kv->pos;
    a.K_new = static_cast<const uint16_t *>(K_new);
    a.V_new = static_cast<const uint16_t *>(V_new);
    a.pos_new = pos_new;
    a.lens = kv->lens;
    a.block_table = kv->block_table;
    a.batch = kv->batch;
    a.n_kv = c->Hkv;
    a.n_layers = kv->n_layers;
    a.page_size = kv->page_size;
    a.max_pages = kv->max_pages;
    a.n_pages = kv->n_pages;
    a.status = c->d_status;
    a.lens_out = kv->lens_out;
    a.pos_adv = advance ? const_cast<int32_t *>(pos_new) : nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // one cluster of cs CTAs per sequence; a programmatic dependent of the launch before it on
    // this stream (in a decode loop, the previous token's append): its launch overlaps that
    // grid's end, and the kernel waits for it before its first memory access
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.gridDim = dim3((unsigned)(kv->batch * cs));
    cfg.blockDim = dim3((unsigned)(tri::kAppendWarps * 32));
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (c->D == 128)
        ce = cudaLaunchKernelEx(&cfg, tri::tri_append_kernel<128>, a);
    else
        ce = cudaLaunchKernelEx(&cfg, tri::tri_append_kernel<64>, a);
    if (ce != cudaSuccess) return cuda_fail(c, ce, "append rows");
    return TRI_OK;
}
}  // namespace

tri_status tri_append(tri_ctx *c, const tri_kv *kv, const void *K_new, const void *V_new, const int32_t *pos_new,
                      void *stream) {
    NvtxRange r("tri_append");
    return append_impl(c, kv, K_new, V_new, pos_new, false, stream);
}

tri_status tri_append_advance(tri_ctx *c, const tri_kv *kv, const void *K_new, const void *V_new, int32_t *pos,
                              void *stream) {
    NvtxRange r("tri_append_advance");
    return append_impl(c, kv, K_new, V_new, pos, true, stream);
}

tri_status tri_set_offset_combine(tri_ctx *c, int combine) {
    if (!c) return TRI_EINVAL;
    if (combine != TRI_OFFSETS_MEAN && combine != TRI_OFFSETS_MAX) return TRI_EINVAL;
    c->combine = combine;
    return TRI_OK;
}

tri_status tri_set_score_engine(tri_ctx *c, int engine) {
    if (!c) return TRI_EINVAL;
    if (engine != TRI_ENGINE_AUTO && engine != TRI_ENGINE_CUDA_CORES && engine != TRI_ENGINE_TENSOR)
        return TRI_EINVAL;
    c->engine = engine;
    return TRI_OK;
}

tri_status tri_set_tuning(tri_ctx *c, int cluster_size, int buffers_per_warp) {
    if (!c) return TRI_EINVAL;
    if (cluster_size != 0 && cluster_size != 1 && cluster_size != 2 && cluster_size != 4 &&
        cluster_size != 8 && cluster_size != 16)
        return TRI_EINVAL;
    if (buffers_per_warp < 0 || buffers_per_warp > 4) return TRI_EINVAL;
    c->tune_cs = cluster_size;
    c->tune_nslot = buffers_per_warp;
    return TRI_OK;
}

tri_status tri_get_error(tri_ctx *c, void *stream, int32_t *detail_code, int64_t *detail_unit) {
    if (detail_code) *detail_code = 0;
    if (detail_unit) *detail_unit = -1;
    if (!c) return TRI_EINVAL;
    if (cudaSetDevice(c->device) != cudaSuccess) return TRI_ECUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TRI_ECUDA;
    unsigned long long v = 0;
    if (cudaMemcpy(&v, c->d_status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return TRI_ECUDA;
    if (v == 0) return TRI_OK;
    if (cudaMemset(c->d_status, 0, sizeof v) != cudaSuccess) return TRI_ECUDA;
    if (detail_code) *detail_code = (int32_t)(v >> 32);
    if (detail_unit) *detail_unit = (int64_t)(uint32_t)(v & 0xffffffffu);
    return TRI_EDEVICE;
}

tri_status tri_get_failed_units(tri_ctx *c, void *stream, int32_t *units, int32_t capacity, int32_t *count) {
    if (count) *count = 0;
    if (!c || capacity < 0 || (capacity > 0 && !units)) return TRI_EINVAL;
    if (cudaSetDevice(c->device) != cudaSuccess) return TRI_ECUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TRI_ECUDA;
    unsigned n = 0;
    if (cudaMemcpy(&n, c->d_fail_count, sizeof n, cudaMemcpyDeviceToHost) != cudaSuccess) return TRI_ECUDA;
    const int listed = (int)std::min<unsigned>(n, (unsigned)std::min(capacity, kFailCap));
    if (listed > 0 &&
        cudaMemcpy(units, c->d_fail_units, sizeof(int32_t) * listed, cudaMemcpyDeviceToHost) != cudaSuccess)
        return TRI_ECUDA;
    if (n > 0 && cudaMemset(c->d_fail_count, 0, sizeof n) != cudaSuccess) return TRI_ECUDA;
    if (count) *count = (int32_t)std::min<unsigned>(n, 0x7fffffffu);
    return TRI_OK;
}

tri_status tri_set_test_fault(tri_ctx *c, int64_t unit, int32_t wait_tries) {
    if (!c) return TRI_EINVAL;
    if (wait_tries < 0 || unit < -1) return TRI_EINVAL;
    c->inject_unit = unit;
    c->wait_tries = wait_tries > 0 ? wait_tries : tri::kWaitTries;
    return TRI_OK;
}

const char *tri_last_error(tri_ctx *c) {
    if (!c) return "no context";
    return c->last_error;
}

const char *tri_status_str(tri_status s) {
    switch (s) {
        case TRI_OK: return "TRI_OK";
        case TRI_EINVAL: return "TRI_EINVAL: invalid argument";
        case TRI_ENOMEM: return "TRI_ENOMEM: allocation failed";
        case TRI_ECUDA: return "TRI_ECUDA: CUDA runtime error";
        case TRI_ESTATE: return "TRI_ESTATE: no calibration statistics loaded";
        case TRI_EDEVICE: return "TRI_EDEVICE: the device flagged a problem";
        case TRI_EUNSUPPORTED: return "TRI_EUNSUPPORTED: unsupported device or size";
    }
    return "unknown tri_status";
}

int tri_version(void) { return 100; }

}  // extern "C"
