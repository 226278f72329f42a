// tri_append.cuh -- the decode loop's write between prunes, for sm_100a.
//
// Pages cited (titles; sections as headed on each page):
//   [10100]    the 10100.com article 127765992 on TriAttention
//   [Summary]  "TriAttention：面向长文本推理的高效KV缓存压缩，2.5倍吞吐提升与10.7倍内存缩减"
//
// Between two prunes ([10100] §TriAttention方法 and [Summary] §方案设计 item 4: once every 128
// generated tokens) every decode step appends the new token's key, value and position to each
// (sequence, layer, KV head) unit of the paged cache, at slot lens[s]. One cluster of CTAs per
// sequence: every unit of a sequence sees the same slot and the same page, so one thread per CTA
// looks them up, the warps move the units' K and V rows (16 bytes per lane) and positions, and
// after a cluster barrier the cluster's first CTA publishes the new length (one launch per
// appended token, each a programmatic dependent of the launch before it).
#pragma once

#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tri {

namespace cg = cooperative_groups;

constexpr int kAppendWarps = 16;      // warps per CTA (512 threads)
constexpr int kAppendMaxCluster = 8;  // CTAs per sequence, at most (the portable cluster size)
constexpr int kAppendBatch = 4;       // units per warp whose rows are loaded before any is stored

// CTAs per sequence for n_units_per_seq = n_layers * n_kv units: one unit per warp where possible.
inline int append_cluster_size(long long n_units_per_seq) {
    const long long need = (n_units_per_seq + kAppendWarps - 1) / kAppendWarps;
    return (int)(need < 1 ? 1 : need > kAppendMaxCluster ? kAppendMaxCluster : need);
}

struct AppendArgs {
    uint16_t *K, *V;              // paged pools [n_layers][n_pages][n_kv][page_size][D]
    int32_t *pos;                 // [n_layers][n_pages][n_kv][page_size]
    const uint16_t *K_new, *V_new;  // [n_layers][batch][n_kv][D]
    const int32_t *pos_new;       // [batch]
    const int32_t *lens;          // [batch]
    int32_t *lens_out;            // [batch] (may be lens itself)
    const int32_t *block_table;   // [batch][max_pages]
    int batch, n_kv, n_layers, page_size, max_pages, n_pages;
    unsigned long long *status;   // first device-detected problem
    int32_t *pos_adv;             // pos_new itself, advanced by one for the accepted sequences (or null)
};

__device__ __forceinline__ void append_record(unsigned long long *st, int code, long long unit) {
    const unsigned long long v = ((unsigned long long)(unsigned)code << 32) | (unsigned long long)(unsigned)unit;
    atomicCAS(st, 0ull, v);
}

// Grid: batch clusters of cs CTAs (launched with that cluster size); cluster c appends to
// sequence c. Unit u = lr * n_kv + g of the sequence goes to warp u mod (cs * kAppendWarps) of
// the cluster, in batches of kAppendBatch units per warp.
template <int D>
__global__ void __launch_bounds__(kAppendWarps * 32) tri_append_kernel(const AppendArgs a) {
    // launched as a programmatic dependent of the grid before it on the stream (usually the
    // previous token's append, which writes the lengths and positions read here): nothing is
    // read before that grid has finished and its writes are visible; the next append may then
    // be scheduled, so at most two appends are in flight
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = (int)cluster.num_blocks();
    const int rank = (int)cluster.block_rank();
    const int s = (int)(blockIdx.x / cs);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per_seq = a.n_layers * a.n_kv;
    const int stride = cs * kAppendWarps;
    constexpr int PIECES = D / 8;  // 16-byte pieces per row; lane p < 2 PIECES moves piece p of K then V
    const bool mover = lane < 2 * PIECES;
    const bool isv = lane >= PIECES;
    const int q = isv ? lane - PIECES : lane;

    uint4 x[kAppendBatch];
    auto load = [&](int u0) {
#pragma unroll
        for (int k = 0; k < kAppendBatch; ++k) {
            const int u = u0 + k * stride;
            if (mover && u < per_seq) {
                const long long src = ((long long)(u / a.n_kv) * a.batch + s) * a.n_kv + u % a.n_kv;
                x[k] = __ldg(reinterpret_cast<const uint4 *>((isv ? a.V_new : a.K_new) + src * D) + q);
            }
        }
    };
    int u0 = rank * kAppendWarps + warp;
    load(u0);  // the source rows do not depend on the slot: in flight during the lookup

    __shared__ int n_s, page_s, bad_s, p_s;
    if (threadIdx.x == 0) {
        const int n = a.lens[s];  // plain loads: lens_out may be lens, pos_adv is pos_new
        const long long cap = (long long)a.page_size * a.max_pages;
        int page = -1, bad = 0;
        if (n < 0 || n >= cap) {
            bad = 1;  // TRI_DEV_LEN_GT_CAP: no slot left for the new token
        } else {
            page = __ldg(a.block_table + (long long)s * a.max_pages + n / a.page_size);
            if (page < 0 || page >= a.n_pages) bad = 2;  // TRI_DEV_BAD_PAGE: the page is not allocated
        }
        n_s = n;
        page_s = page;
        bad_s = bad;
        p_s = a.pos_new[s];
    }
    __syncthreads();
    const int n = n_s, bad = bad_s;
    if (!bad) {
        const long long page_row = (long long)page_s * a.n_kv;
        const int slot = n % a.page_size;
        for (;;) {
#pragma unroll
            for (int k = 0; k < kAppendBatch; ++k) {
                const int u = u0 + k * stride;
                if (u < per_seq) {
                    const long long row =
                        (((long long)(u / a.n_kv) * a.n_pages * a.n_kv + page_row) + u % a.n_kv) * a.page_size + slot;
                    if (mover) reinterpret_cast<uint4 *>((isv ? a.V : a.K) + row * D)[q] = x[k];
                    if (lane == 0) a.pos[row] = p_s;
                }
            }
            u0 += kAppendBatch * stride;
            if (u0 >= per_seq) break;
            load(u0);
        }
    }
    // every CTA of the cluster has read lens[s] and pos_new[s]: the length (and, when asked, the
    // next position) can be published; a refused sequence keeps both
    cluster.sync();
    if (rank == 0 && threadIdx.x == 0) {
        if (bad) {
            append_record(a.status, bad, (long long)s * a.n_kv);  // unit (layer 0, s, head 0)
            a.lens_out[s] = n;
        } else {
            a.lens_out[s] = n + 1;
            if (a.pos_adv) a.pos_adv[s] = p_s + 1;  // the next token's position
        }
    }
}
}  // namespace tri
