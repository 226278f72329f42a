// tri_append.cuh -- the decode loop's write between prunes, for sm_100a.
//
// Pages cited (titles; sections as headed on each page):
//   [10100]    the 10100.com article 127765992 on TriAttention
//   [Summary]  "TriAttention：面向长文本推理的高效KV缓存压缩，2.5倍吞吐提升与10.7倍内存缩减"
//
// Between two prunes ([10100] §TriAttention方法 and [Summary] §方案设计 item 4: once every 128
// generated tokens) every decode step appends the new token's key, value and position to each
// (sequence, layer, KV head) unit of the paged cache, at slot lens[s]. One warp moves one unit's
// K row and V row (16 bytes per lane) and its position; the last CTA to finish advances the
// lengths of the sequences whose rows all went in (one launch per appended token, each a
// programmatic dependent of the launch before it).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tri {

constexpr int kAppendWarps = 8;  // units per CTA

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
    int32_t *seq_bad;             // [batch] refused sequences
    unsigned *done;               // completed-CTA counter (zero between launches)
    int32_t *pos_adv;             // pos_new itself, advanced by one for the accepted sequences (or null)
};

__device__ __forceinline__ void append_record(unsigned long long *st, int code, long long unit) {
    const unsigned long long v = ((unsigned long long)(unsigned)code << 32) | (unsigned long long)(unsigned)unit;
    atomicCAS(st, 0ull, v);
}

// One warp per unit (layer lr, sequence s, KV head g); the last CTA publishes the lengths.
template <int D>
__global__ void __launch_bounds__(kAppendWarps * 32) tri_append_kernel(const AppendArgs a) {
    // launched as a programmatic dependent of the grid before it on the stream (usually the
    // previous token's append, which writes the lengths, positions and counter read here):
    // nothing is read before that grid has finished and its writes are visible; the next
    // append may then be scheduled, so at most two appends are in flight
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
    const long long n_units = (long long)a.n_layers * a.batch * a.n_kv;
    if (unit < n_units) {
        const int g = (int)(unit % a.n_kv);
        const int s = (int)((unit / a.n_kv) % a.batch);
        const int lr = (int)(unit / ((long long)a.n_kv * a.batch));
        const int n = a.lens[s];  // plain load: lens_out may be lens, written at the end of this launch
        const long long cap = (long long)a.page_size * a.max_pages;
        int page = -1;
        int bad = 0;
        if (n < 0 || n >= cap) {
            bad = 1;  // TRI_DEV_LEN_GT_CAP: no slot left for the new token
        } else {
            page = __ldg(a.block_table + (long long)s * a.max_pages + n / a.page_size);
            if (page < 0 || page >= a.n_pages) bad = 2;  // TRI_DEV_BAD_PAGE: the page is not allocated
        }
        if (bad) {
            if (lane == 0) {
                append_record(a.status, bad, unit);
                atomicExch(a.seq_bad + s, 1);
            }
        } else {
            const long long row =
                (((long long)lr * a.n_pages + page) * a.n_kv + g) * a.page_size + n % a.page_size;
            const long long src = ((long long)lr * a.batch + s) * a.n_kv + g;
            constexpr int PIECES = D / 8;  // 16-byte pieces per row
            for (int p = lane; p < 2 * PIECES; p += 32) {
                const bool isv = p >= PIECES;
                const int q = isv ? p - PIECES : p;
                const uint4 x = __ldg(reinterpret_cast<const uint4 *>((isv ? a.V_new : a.K_new) + src * D) + q);
                reinterpret_cast<uint4 *>((isv ? a.V : a.K) + row * D)[q] = x;
            }
            if (lane == 0) a.pos[row] = __ldg(a.pos_new + s);
        }
    }
    // lens_out[s] = lens[s] + 1 for every sequence whose rows all went in (and, when asked, its
    // next position pos_new[s] + 1); refused sequences keep both and their flag is cleared for
    // the next call. Done by the last CTA to finish, after every CTA has read the lengths and
    // positions and raised its flags.
    __shared__ int last_s;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        last_s = atomicAdd(a.done, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (last_s) {
        __threadfence();
        for (int s = threadIdx.x; s < a.batch; s += blockDim.x) {
            const int n = a.lens[s];
            const int refused = atomicExch(a.seq_bad + s, 0);
            a.lens_out[s] = refused ? n : n + 1;
            if (a.pos_adv && !refused) a.pos_adv[s] += 1;  // the next token's position
        }
        if (threadIdx.x == 0) atomicExch(a.done, 0u);
    }
}
}  // namespace tri
