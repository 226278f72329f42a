/*
 * tri.h -- C ABI of the B200 (sm_100a) TriAttention KV-cache scoring-and-pruning pass.
 *
 * Pages cited (titles; sections as headed on each page):
 *   [Deep-dive]  "TriAttention深度解析：用三角函数革命性压缩KV Cache，让长推理从「显存地狱」中脱困"
 *                (chenxutan.com/d/2624)
 *   [Stage]      "旋转舞台上的追光者——TriAttention如何用三角函数破解长文本推理的内存困局"
 *                (zhichai.net/topic/177169654)
 *   [10100]      the 10100.com article 127765992 on TriAttention (untitled extract)
 *   [Summary]    "TriAttention：面向长文本推理的高效KV缓存压缩，2.5倍吞吐提升与10.7倍内存缩减"
 *                (watermelonwater.tech)
 *
 * The pass, per unit = one (sequence s, layer l, KV head g) slice of the cache:
 *   score   s_h(i) = mean_{delta in D} sum_f |qbar_f| |k_f| cos(omega_f (t + delta - p_i) + phi_f)
 *                    + sum_f (1 - R_f) E|q_f| |k_f|
 *           for each of the G query heads h that share KV head g
 *           ([Stage] §TriAttention：把理论变成算法 items 1-2; [10100] §TriAttention方法;
 *            offsets D of [Deep-dive] §3.3); tri_set_offset_combine switches the mean over
 *           delta to the maximum ([Deep-dive] §3.3 and its §4.2 scoring code),
 *   z/max   z-score each head over the unit's keys, max over the G heads
 *           ([10100] §TriAttention方法; [Summary] §方案设计 item 4),
 *   select  keep the B keys with the largest max-z, ties to the lower slot,
 *   compact move the kept K, V and position rows, in their original order, to
 *           slots 0..min(N,B)-1 of the same unit ([Deep-dive] §4 prune_kv_cache),
 * run by the caller once every 128 generated tokens ([10100] §TriAttention方法;
 * [Summary] §方案设计 item 4).
 *
 * Conventions for every entry point:
 *   - Device pointers are plain CUDA device addresses of memory the caller owns.
 *     The library never frees, resizes or retains them past the call.
 *   - `stream` is a cudaStream_t passed as void*. Every launch goes on it;
 *     calls return as soon as the work is enqueued (asynchronous).
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns TRI_EINVAL (or TRI_ESTATE / TRI_EUNSUPPORTED) and launches
 *     nothing. Problems only the device can see are recorded in the context's
 *     device status word and read with tri_get_error. Kernels never trap.
 *     Two kinds:
 *       sequence-level  a length above the capacity, a page id outside the pool, a
 *                       cached position not below t. A validation kernel decides them
 *                       before any unit of the call is touched, so every unit of the
 *                       sequence is left untouched and lens_out[s] = lens[s].
 *       unit-level      a bounded wait that ran out, or a selection that did not give
 *                       exactly min(len, B) keys. That unit is left uncompacted; the
 *                       sequence's other units are pruned and lens_out[s] = min(len, B), so
 *                       the uncompacted unit then holds its first min(len, B) original rows
 *                       (a consistent cache, ascending positions, but not the method's
 *                       choice of keys). A group of CTAs whose wait ran out no longer trusts
 *                       its copy pipeline: it also refuses the one unit it had already taken
 *                       and takes no more (units are handed out dynamically, so other groups
 *                       process the rest). In the tensor-core scoring kernel (max over
 *                       offsets, tensor-core engine) a wait that ran out ends that CTA's tile
 *                       range, and every unit the range touches is refused.
 *                       tri_get_failed_units lists every such unit.
 *   - A context is bound to one device and is not thread-safe: serialise calls
 *     that share a context. Calls that share a context but run on different
 *     streams must not overlap on the GPU (they share the status word, the
 *     completion counter and the scratch that tri_prune, tri_score and
 *     tri_calibrate_estimate use).
 */
#ifndef TRI_H_
#define TRI_H_

#include <stdint.h>

#if defined(__GNUC__)
#define TRI_API __attribute__((visibility("default")))
#else
#define TRI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TRI_OK = 0,
    TRI_EINVAL = 1,       /* bad argument; nothing was launched */
    TRI_ENOMEM = 2,       /* device or host allocation failed */
    TRI_ECUDA = 3,        /* a CUDA runtime call failed */
    TRI_ESTATE = 4,       /* no calibration statistics loaded */
    TRI_EDEVICE = 5,      /* the device flagged bad input or a timed-out wait (tri_get_error) */
    TRI_EUNSUPPORTED = 6  /* not an sm_100 device, or sizes beyond the on-chip limits */
} tri_status;

typedef enum {
    TRI_ROPE_HALF = 0,        /* band f = dims (f, f + d/2): Qwen / NeoX rotary layout */
    TRI_ROPE_INTERLEAVED = 1  /* band f = dims (2f, 2f + 1): GPT-J rotary layout */
} tri_rope_layout;

/* How the future offsets delta combine in the trigonometric score (tri_set_offset_combine). */
typedef enum {
    TRI_OFFSETS_MEAN = 0,  /* mean over delta (default): folds into one coefficient per band */
    TRI_OFFSETS_MAX = 1    /* max over delta ([Deep-dive] §3.3 and its §4.2 scoring code) */
} tri_offset_combine;

/* Which kernels score the mean mode (tri_set_score_engine). */
typedef enum {
    TRI_ENGINE_AUTO = 0,        /* tensor cores at group 8, CUDA cores below (the default) */
    TRI_ENGINE_CUDA_CORES = 1,  /* one fused launch: folded dot products on the CUDA cores */
    TRI_ENGINE_TENSOR = 2       /* tcgen05 scoring kernel, then the fused select and compaction */
} tri_score_engine;

/* Device-side problem codes reported by tri_get_error in *detail_code. */
enum {
    TRI_DEV_NONE = 0,
    TRI_DEV_LEN_GT_CAP = 1,   /* lens[s] < 0 or above the unit capacity */
    TRI_DEV_BAD_PAGE = 2,     /* a block-table entry outside [0, n_pages) */
    TRI_DEV_TIMEOUT = 3,      /* a bounded wait on an asynchronous copy gave up (unit-level) */
    TRI_DEV_INTERNAL = 4,     /* the selection did not produce exactly min(len, B) keys (unit-level) */
    TRI_DEV_T_NOT_AFTER_POS = 5  /* a unit's last cached position is not below t (sequence-level) */
};

typedef struct tri_ctx tri_ctx;   /* opaque: device statistics, status word, counters */

/*
 * The cache one call works on. All pointers are device pointers owned by the caller.
 *
 * Dense layout (block_table == NULL):
 *   K, V  bf16 [n_layers][batch][n_kv_heads][cap][head_dim]   (16-byte aligned)
 *   pos   int32 [n_layers][batch][n_kv_heads][cap]            ascending within a unit
 * Paged layout (block_table != NULL), one pool per layer, shared block table:
 *   K, V  bf16 [n_layers][n_pages][n_kv_heads][page_size][head_dim]
 *   pos   int32 [n_layers][n_pages][n_kv_heads][page_size]
 *   block_table int32 [batch][max_pages]: logical page j of sequence s lives in
 *         pool page block_table[s][j]; a unit's capacity is max_pages * page_size.
 * lens      int32 [batch]: cached tokens of each sequence (same for every layer and
 *           KV head), read only.
 * lens_out  int32 [batch] or NULL: receives min(lens[s], budget) after tri_prune for
 *           every sequence the device accepted (may alias lens). Pass NULL when a
 *           cache is pruned in several layer chunks and update lens after the last.
 * layer_begin, n_layers: the layers this call covers, indexing the loaded statistics;
 *           the buffers above hold exactly these n_layers layers.
 * n_kv_heads and head_dim come from the loaded statistics.
 */
typedef struct {
    void *K;
    void *V;
    int32_t *pos;
    const int32_t *lens;
    int32_t *lens_out;
    const int32_t *block_table;
    int32_t batch;
    int32_t cap;          /* dense: slots per unit; ignored when paged */
    int32_t page_size;    /* paged: tokens per page, a multiple of 16; ignored when dense */
    int32_t max_pages;    /* paged: block-table row length */
    int32_t n_pages;      /* paged: pages in each layer's pool */
    int32_t layer_begin;
    int32_t n_layers;
} tri_kv;

/* Create a context on CUDA device `device` (must be compute capability 10.0).
 * Allocates about 16 KB of device memory (status word, completion counter, the list of units
 * left uncompacted by unit-level failures). */
TRI_API tri_status tri_create(tri_ctx **out, int device);

/* Release the context and everything it allocated. NULL is accepted. */
TRI_API tri_status tri_destroy(tri_ctx *ctx);

/*
 * Load calibration statistics (host fp32 arrays, copied; the caller keeps ownership).
 *   q_mean       [n_layers][n_kv_heads*group][head_dim]  pre-RoPE query centre qbar, in the
 *                same dim layout as the keys ([Deep-dive] §3.4; [Stage] item 1: E[q_f])
 *   q_norm_mean  [n_layers][n_kv_heads*group][head_dim/2] E|q_f| per band ([Stage] item 2)
 *   R            [n_layers][n_kv_heads*group][head_dim/2] concentration R_f = |E q_f| / E|q_f|
 *                ([Stage] §破局之道)
 *   offsets      [n_offsets] future offsets delta ([Deep-dive] §3.3: 1, 2, 4, ..., 2^16)
 * Query head h belongs to KV head h / group. head_dim in {64, 128}; group in {1, 2, 4, 8};
 * rope_base > 0; all values finite. The per-band constants (omega_f, the offset average
 * A_f = mean_delta e^{i omega_f delta}, qbar_f * A_f and (1 - R_f) E|q_f|) are formed
 * here in fp64. Replaces any statistics loaded before. Synchronous.
 */
TRI_API tri_status tri_calibrate_load(tri_ctx *ctx, int n_layers, int n_kv_heads, int group, int head_dim,
                              double rope_base, tri_rope_layout layout,
                              const float *q_mean, const float *q_norm_mean, const float *R,
                              const int64_t *offsets, int n_offsets);

/*
 * Append one token to every sequence of a paged cache: the decode loop's write between two
 * prunes, which the caller runs once every 128 generated tokens ([10100] §TriAttention方法;
 * [Summary] §方案设计 item 4).
 *   kv       paged cache (block_table required); its n_layers layers, lens and lens_out
 *   K_new, V_new  bf16 [n_layers][batch][n_kv_heads][head_dim] device, 16-byte aligned: the
 *            new token's key and value rows (the key after RoPE, like the cached ones)
 *   pos_new  int32 [batch] device: the new token's position in each sequence
 * Slot lens[s] of every unit of sequence s receives the rows and the position, and
 * lens_out[s] = lens[s] + 1 (lens_out may alias lens; it is required here). The page that
 * slot lands in, block_table[s][lens[s] / page_size], must already be allocated by the
 * caller (an id in [0, n_pages)); freeing the pages past a sequence's length after a prune
 * is the caller's business too. A sequence whose slot is past its capacity or lands in an
 * unallocated page is refused as a whole (lens_out[s] = lens[s]; tri_get_error reports
 * TRI_DEV_LEN_GT_CAP or TRI_DEV_BAD_PAGE): every unit of a sequence sees the same slot and
 * page, so a refused sequence receives no row. Needs the statistics loaded (for n_kv_heads
 * and head_dim).
 * One launch on `stream` (a cluster of CTAs per sequence, whose first CTA writes lens_out[s]
 * after the cluster's barrier), a programmatic dependent of the work before it on the stream:
 * its launch may overlap the end of the kernel before it, but it reads and writes nothing until
 * that kernel has finished, so stream order holds as for a plain launch. tri_get_error reports
 * a refused sequence s as unit s * n_kv_heads (its first layer and KV head).
 */
TRI_API tri_status tri_append(tri_ctx *ctx, const tri_kv *kv, const void *K_new, const void *V_new,
                              const int32_t *pos_new, void *stream);

/*
 * tri_append for a decode loop whose next token position follows the last one: the same append
 * of the rows and of the position pos[s], after which pos[s] += 1 for every sequence that
 * accepted the token (a refused sequence keeps its position as it keeps its length). The
 * caller's per-step position update is thereby part of the same single launch.
 *   pos      int32 [batch] device: in, the new token's positions; out, the next ones
 * Everything else as tri_append.
 */
TRI_API tri_status tri_append_advance(tri_ctx *ctx, const tri_kv *kv, const void *K_new, const void *V_new,
                                      int32_t *pos, void *stream);

/*
 * Estimate the calibration statistics from pre-RoPE query samples (the pages' offline
 * calibration step: [Deep-dive] §3.4; the statistics of [Stage] §TriAttention：把理论变成算法
 * items 1-2 and the concentration of [Stage] §破局之道, taken per band).
 *   Q            bf16 [n_layers][T][n_q_heads][head_dim] device: the pre-RoPE queries of T
 *                calibration tokens, dims in the keys' rotary layout `layout`
 *   q_mean       fp32 [n_layers][n_q_heads][head_dim] device, written: E[q_f] over the T tokens
 *                (real part at band f's first dim, imaginary part at its second)
 *   q_norm_mean  fp32 [n_layers][n_q_heads][head_dim/2] device, written: E|q_f|
 *   R            fp32 [n_layers][n_q_heads][head_dim/2] device, written: |E[q_f]| / E|q_f|,
 *                0 for a band whose samples are all zero
 * The three outputs are what tri_calibrate_load takes (after a copy to the host).
 * Sums run in fp64 (|q_f| from the exact bf16 components with one fp32 rounding of
 * re^2 + im^2 and a correctly rounded fp32 square root) in a fixed order, so the results do
 * not depend on the GPU; the outputs are rounded to fp32 once. Runs on `stream` (two launches);
 * Q is only read. head_dim in {64, 128}; T, n_layers, n_q_heads >= 1; Q 16-byte aligned.
 * Uses the context's scratch (grown with a device-synchronising cudaMalloc when a call needs
 * more than any call before: n_layers * n_q_heads * head_dim/2 * ceil(T / 256) * 24 bytes).
 * Does not need statistics to be loaded. Errors: TRI_EINVAL (argument), TRI_EUNSUPPORTED
 * (head_dim, sizes), TRI_ENOMEM, TRI_ECUDA (tri_last_error says which call failed).
 */
TRI_API tri_status tri_calibrate_estimate(tri_ctx *ctx, const void *Q, int n_layers, int T, int n_q_heads,
                                          int head_dim, tri_rope_layout layout, float *q_mean,
                                          float *q_norm_mean, float *R, void *stream);

/*
 * Score every cached key and prune each unit to its top `budget` keys, in place.
 *   t       int32 [batch] device: current query position of each sequence; the
 *           future queries are at t + delta. Positions in the cache must be < t: a
 *           sequence with a unit whose last cached position is >= t is refused
 *           (TRI_DEV_T_NOT_AFTER_POS, sequence-level).
 *   budget  B >= 1 keys kept per unit.
 * After the call (in stream order) slots [0, min(len, B)) of every unit hold the kept
 * K, V and position rows in ascending original order; slots at or beyond that are
 * left as they were (reclaiming them is the caller's business); units with len <= B
 * are not touched at all. lens_out receives the new lengths.
 */
TRI_API tri_status tri_prune(tri_ctx *ctx, const tri_kv *kv, const int32_t *t, int32_t budget, void *stream);

/*
 * tri_prune without any device allocation at call time. (The TriAttention pages have no
 * counterpart: this is an interface for callers that cannot allocate device memory while they
 * run, e.g. a serving loop whose device memory belongs to another allocator, or one that cannot
 * afford the device-wide synchronisation of the cudaFree that tri_prune performs when it grows
 * its scratch.)
 *   Same arguments, semantics and results as tri_prune. The scores of the units in flight live
 *   in a fixed 64 MiB device array that the library holds on every GPU that loads it, until the
 *   process exits; the validation kernel writes every sequence's verdict (0 when accepted) into
 *   a fixed array of 16384 entries on every call, so nothing needs clearing beforehand. It
 *   calls no cudaMalloc, cudaFree or allocating library routine.
 * Limits: batch <= 16384; the unit-capacity limit of tri_prune applies unchanged (within it
 *   one unit's score slot, capacity * (group + 1) floats, stays below 19 MB). When the 64 MiB
 *   holds fewer slots than tri_prune would run clusters, fewer clusters run: same results, a
 *   longer run. Sizes beyond the limits return TRI_EUNSUPPORTED and tri_last_error says why;
 *   nothing is launched.
 * The first call on a device looks up the arrays' device addresses (cudaGetSymbolAddress);
 *   make that first call before any stream capture. Every call shares the two arrays and
 *   leaves its contents there: calls that overlap on the GPU (other streams, other contexts on
 *   the same device) race on them and must be serialised by the caller.
 */
TRI_API tri_status tri_prune_noalloc(tri_ctx *ctx, const tri_kv *kv, const int32_t *t, int32_t budget,
                                     void *stream);

/*
 * Decode attention over a (pruned) cache: the consumer of the compacted cache. For every query
 * head h of every unit, out_h = sum_i softmax_i(q_h . k_i / sqrt(head_dim)) v_i over the unit's
 * cached rows [0, lens[s]) (the page "TriAttention 深度解析：MIT韩松团队如何用三角函数让单卡
 * 4090跑出百万Token上下文" writes this attention out in its section 二, TriAttention的核心发现).
 * The query is post-RoPE like the stored keys, so each logit depends on the distance only and
 * the kept keys' non-contiguous positions need no other treatment.
 *   kv    the cache (dense or paged, as for tri_prune): K, V, lens, block table and layer range
 *         are read; pos, lens_out are not used
 *   q     bf16 [n_layers][batch][n_kv_heads*group][head_dim] device, 16-byte aligned: the
 *         post-RoPE queries of the current decode step, one per query head
 *   out   fp32 [n_layers][batch][n_kv_heads*group][head_dim] device, written
 * Each K and V row is read once (HBM-bound); logits, the softmax and the weighted sum run in
 * fp32 (exponentials in base 2 with the scale folded into the query). A sequence with lens 0
 * gets zeros. Sequences refused by the sequence-level checks (length above the capacity, a page
 * outside the pool; TRI_EDEVICE through tri_get_error) are not written. When there are too few
 * units to fill the GPU, a unit's rows are split into chunks whose partial results a second
 * launch merges; the partials live in the context's scratch, grown on demand (a synchronising
 * cudaMalloc when a call needs more than any call before). Needs the statistics loaded (for
 * n_kv_heads, group and head_dim). Errors: TRI_EINVAL, TRI_ESTATE, TRI_EUNSUPPORTED, TRI_ENOMEM,
 * TRI_ECUDA.
 */
TRI_API tri_status tri_decode_attention(tri_ctx *ctx, const tri_kv *kv, const void *q, float *out, void *stream);

/*
 * Debug / parity entry: score without pruning.
 *   raw   float [n_layers][batch][n_kv_heads*group][cap_u] or NULL: s_h(i) per query head
 *   zmax  float [n_layers][batch][n_kv_heads][cap_u] or NULL: max over the group of z_h(i)
 * where cap_u is cap (dense) or max_pages*page_size (paged), indexed by logical slot.
 * Slots at or beyond lens[s] are not written. The cache is not modified; lens_out is ignored.
 * pos may be NULL here; when it is given, positions are checked against t as in tri_prune.
 * Sequences refused by the sequence-level checks are not written at all.
 */
TRI_API tri_status tri_score(tri_ctx *ctx, const tri_kv *kv, const int32_t *t, float *raw, float *zmax,
                     void *stream);

/*
 * Synchronise `stream`, read and clear the context's device status word.
 * Returns TRI_OK, or TRI_EDEVICE with the first problem's code (TRI_DEV_*) and the
 * unit index u = (layer_in_call * batch + s) * n_kv_heads + g it was seen on
 * (either out-pointer may be NULL).
 */
TRI_API tri_status tri_get_error(tri_ctx *ctx, void *stream, int32_t *detail_code, int64_t *detail_unit);

/*
 * Synchronise `stream`, then read and clear the list of units that unit-level failures
 * (TRI_DEV_TIMEOUT, TRI_DEV_INTERNAL) left uncompacted since the list was last read.
 *   units     int32 host array of `capacity` entries, written with up to `capacity` unit
 *             indices (as in tri_get_error), in no particular order; may be NULL when
 *             capacity is 0
 *   count     receives how many failures were recorded, which may exceed what was listed:
 *             the device keeps the first 4096
 * Device-detected sequence-level problems are not listed (tri_get_error reports them).
 */
TRI_API tri_status tri_get_failed_units(tri_ctx *ctx, void *stream, int32_t *units, int32_t capacity,
                                        int32_t *count);

/*
 * Test hook for the failure path (not part of the paper's pass; off by default).
 *   unit        index (as in tri_get_error) of a unit whose first key copy the scoring kernels
 *               arm but never issue on the next calls, so that the wait for it runs out; -1 = off
 *   wait_tries  tries of the bounded waits, about 1 ms each (0 = the default 1024); the fused
 *               CUDA-core kernel's key-stream wait keeps the default bound (about one second)
 * The withheld copy never lands, the wait gives up after wait_tries tries, the kernel records
 * TRI_DEV_TIMEOUT and leaves the affected units uncompacted (unit-level failure); no copy is
 * left in flight and nothing waits without bound.
 */
TRI_API tri_status tri_set_test_fault(tri_ctx *ctx, int64_t unit, int32_t wait_tries);

/*
 * Launch-shape override for measurement and tests (not part of the paper's pass).
 *   cluster_size      CTAs that share one unit: 1, 2, 4, 8 or 16; 0 = automatic
 *                     (the smallest that holds the unit's scores on chip while giving
 *                     the GPU at least two CTAs per SM).
 *   buffers_per_warp  key-streaming buffers per warp, 1..4; 0 = automatic (2).
 * Sizes that do not fit on chip with the requested shape make tri_prune / tri_score
 * return TRI_EUNSUPPORTED.
 */
TRI_API tri_status tri_set_tuning(tri_ctx *ctx, int cluster_size, int buffers_per_warp);

/*
 * Choose how later tri_prune / tri_score calls on this context combine the future offsets.
 *   TRI_OFFSETS_MEAN  s_h = mean over delta of S_trig + S_norm. The mean folds into one
 *                     complex coefficient per band (A_f), so a key costs one dot product per
 *                     head. The default.
 *   TRI_OFFSETS_MAX   s_h = max over delta of S_trig + S_norm: the reading of [Deep-dive] §3.3
 *                     (score at every offset of the geometric set, keep the largest) and of
 *                     its §4.2 scoring code, which then adds the norm score. This does not
 *                     fold: every key needs group * n_offsets dot products, run as a
 *                     tensor-core contraction (the bf16 keys against a hi + lo bf16 split of
 *                     the fp64 coefficients qbar_f e^{i omega_f (t + delta)}, fp32
 *                     accumulation), followed by the same z-score, max over the group,
 *                     top-B select and compaction.
 * Everything else (arguments, results, in-place semantics, device status codes) is the same
 * in both modes. The max mode needs group * n_offsets <= 256 (else the call returns
 * TRI_EUNSUPPORTED) and scratch that tri_prune / tri_score grow on demand: the scores of up
 * to 1 GiB worth of layers at a time (n_layers_chunk * batch * n_kv_heads * cap_u * group * 4
 * bytes; longer calls run in chunks of layers), one coefficient image per unit of a chunk
 * (42 KB at head_dim 128, group 4, 17 offsets) and small tables. tri_prune_noalloc supports
 * the mean only (TRI_EUNSUPPORTED in max mode). Errors: TRI_EINVAL (NULL context, unknown
 * mode).
 * The max mode's scoring kernel runs one CTA per SM and allocates up to 512 columns of tensor
 * memory per CTA with a blocking allocation: do not run it concurrently (on another stream)
 * with other kernels that hold tensor memory on the same device, or its allocation may wait
 * until they release theirs.
 */
TRI_API tri_status tri_set_offset_combine(tri_ctx *ctx, int combine);

/*
 * Choose the kernels that score the mean mode on later tri_prune / tri_score calls (the max mode
 * always uses the tensor cores; tri_prune_noalloc always the fused CUDA-core kernel).
 *   TRI_ENGINE_CUDA_CORES  one fused launch per call: each key's folded dot products and norm
 *                          terms on the CUDA cores (fp32), z-score, select and compaction on chip.
 *   TRI_ENGINE_TENSOR      the tcgen05 kernel of the max mode with one column per head, whose
 *                          coefficient is qbar A_f e^{i omega_f t} (the offset average folded in,
 *                          as a hi + lo bf16 pair), writes the scores (group * 4 bytes per key,
 *                          scratch grown on demand); then the fused kernel z-scores, selects and
 *                          compacts. Worth it where the CUDA cores cannot keep up with HBM
 *                          (group 8: about 13 flop per key byte).
 *   TRI_ENGINE_AUTO        tensor cores at group 8, the fused kernel otherwise (the default).
 * Results agree within the score tolerance (1e-4 of a head's largest score). Errors:
 * TRI_EINVAL (NULL context, unknown engine).
 */
TRI_API tri_status tri_set_score_engine(tri_ctx *ctx, int engine);

/* Tracing: tri_prune, tri_prune_noalloc, tri_score, tri_calibrate_estimate and tri_append each
 * mark their host-side span (argument checks and launches) with an NVTX range in the domain
 * "tri"; the max-over-offsets mode adds one range per chunk of layers. A timeline profiler shows
 * them; without one they cost a few nanoseconds. */

/* Text of the last host-side failure on this context (the CUDA error and the call that
 * returned it), or an empty string. Valid until the next call on the context. */
TRI_API const char *tri_last_error(tri_ctx *ctx);

/* Static, human-readable name of a status. */
TRI_API const char *tri_status_str(tri_status s);

/* Library version: major * 10000 + minor * 100 + patch. */
TRI_API int tri_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TRI_H_ */
