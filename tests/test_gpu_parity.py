"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle, element by element.

Small caches are drawn on the CPU from a seed, copied to the device, scored and pruned
there, and every unit is compared with the oracle run on the same bits: raw scores,
max-z, kept sets (up to threshold ties), compacted rows (bit-exact), lengths, and the
slots the prune must not touch.
"""
import numpy as np
import pytest
import torch

import tri_synth as ts
import gpu_util as gu
from rope_aware_key_tri_b200 import tri

pytestmark = pytest.mark.gpu


def _snapshot(cache):
    return cache.K.clone(), cache.V.clone(), cache.pos.clone()


def _same(a, b):
    """Bitwise equality (the caches hold NaN fill beyond each sequence's length)."""
    if a.dtype == torch.bfloat16:
        a, b = a.view(torch.int16), b.view(torch.int16)
    return torch.equal(a, b)


def _written_mask_dense(cache, M_of_seq):
    """Bool [L][batch][Hkv][cap]: slots a prune may write (dst slots [0, M) per unit)."""
    s = cache.spec
    m = torch.zeros((s.n_layers, s.batch, s.n_kv_heads, cache.cap), dtype=torch.bool, device="cuda")
    for b in range(s.batch):
        m[:, b, :, :M_of_seq[b]] = True
    return m


def full_parity(cache, budget=None, cluster_size=0, check_scores=True, label="", combine="mean", engine="auto"):
    s = cache.spec
    B = s.budget if budget is None else budget
    ctx = gu.context_for(cache, cluster_size, combine=combine, engine=engine)
    if check_scores:
        raw, zmx = gu.gpu_score(ctx, cache)
    rows_in = [cache.unit_rows(u) for u in range(cache.n_units)]
    lens_before = cache.lens_host.copy()
    K0, V0, P0 = _snapshot(cache)
    st, code, unit = gu.gpu_prune(ctx, cache, B)
    assert st == tri.TRI_OK, (st, code, unit)
    M_of_seq = np.minimum(lens_before, B)
    assert np.array_equal(cache.lens_host, M_of_seq)
    swaps = 0
    for u in range(cache.n_units):
        l, b, g = cache.unit_index(u)
        lab = f"{label} unit {u} (l={l}, s={b}, g={g}, N={lens_before[b]})"
        orc = gu.oracle_unit(cache, u, B, rows=rows_in[u], combine=combine)
        if check_scores:
            gu.check_scores(raw[l, b, g * s.group:(g + 1) * s.group], zmx[l, b, g], orc, lab)
        out = cache.unit_rows(u)
        kept = gu.kept_from_output(rows_in[u][2], out[2])
        swaps += gu.check_kept(kept, orc, B, lab)
        gu.check_compacted(rows_in[u], out, kept, lab)
        if check_scores:
            gu.self_consistent_select(zmx[l, b, g, :lens_before[b]], kept, B, lab)
    # nothing outside the destination slots [0, M) of each unit changed
    if not cache.paged:
        m = _written_mask_dense(cache, M_of_seq)
        assert _same(cache.K[~m], K0[~m]) and _same(cache.V[~m], V0[~m])
        assert _same(cache.pos[~m], P0[~m])
    else:
        ps = s.page_size
        bt = cache.block_table_host
        written = torch.zeros(cache.pos.shape, dtype=torch.bool, device="cuda")
        for b in range(s.batch):
            for j in range(M_of_seq[b]):
                written[:, int(bt[b, j // ps]), :, j % ps] = True
        assert _same(cache.K[~written], K0[~written]) and _same(cache.V[~written], V0[~written])
        assert _same(cache.pos[~written], P0[~written])
    ctx.close()
    return swaps


def _small(name, **kw):
    return ts.replace(ts.WORKLOADS[name], **kw)


def test_tiny_d64_n256_full():
    cache = ts.make_cache(ts.WORKLOADS["tiny_d64_n256"], 0).to("cuda")
    full_parity(cache, label="tiny")


@pytest.mark.parametrize("engine", ["cuda_cores", "tensor"])
@pytest.mark.parametrize("layout", [ts.HALF, ts.INTERLEAVED], ids=["half", "interleaved"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_shapes(head_dim, group, layout, engine):
    """Both engines of the mean mode: the fused CUDA-core kernel and the tensor-core scoring
    kernel (one column per head carrying the folded offset average) followed by the fused
    select and compaction."""
    spec = ts.CacheSpec(name="shapes", head_dim=head_dim, group=group, n_kv_heads=2, n_layers=2, batch=2,
                        rope_base=1e6 if head_dim == 128 else 1e4, budget=200,
                        offsets=ts.pow2_offsets(16), positions="end_at_t", lens=(301, 517),
                        t=(9000, 700), key_sigma=(0.1, 0.6), layout=layout, cap=640)
    cache = ts.make_cache(spec, 11 + head_dim + group + 7 * layout).to("cuda")
    full_parity(cache, label=f"d{head_dim} G{group} L{layout} {engine}", engine=engine)


@pytest.mark.parametrize("cluster_size", [1, 2, 4, 8, 16])
def test_cluster_sizes(cluster_size):
    spec = ts.CacheSpec(name="cs", head_dim=128, group=4, n_kv_heads=2, n_layers=1, batch=3,
                        rope_base=1e6, budget=333, offsets=ts.pow2_offsets(16), positions="periodic",
                        lens=(1501, 1000, 334), t=(20000, 5000, 900), key_sigma=(0.1, 0.6), recent=128)
    cache = ts.make_cache(spec, 5).to("cuda")
    full_parity(cache, cluster_size=cluster_size, label=f"cs{cluster_size}")


@pytest.mark.parametrize("engine", ["cuda_cores", "tensor"])
@pytest.mark.parametrize("page_size", [16, 48, 64])  # 48: not a power of two (division path)
def test_paged_permuted(page_size, engine):
    spec = _small("qwen3_32b_paged_ragged", n_layers=2, batch=3, lens=(700, 129, 513), page_size=page_size,
                  budget=128, cap=1024)
    cache = ts.make_cache(spec, 3).to("cuda")
    full_parity(cache, label=f"paged{page_size} {engine}", engine=engine)


def test_qwen3_8b_decode_b16_2176_full():
    """Single-layer decode-time prune, batch 16, 2176 -> 2048, every unit against the oracle."""
    import oracle
    spec = ts.WORKLOADS["qwen3_8b_decode_b16_2176"]
    cache = ts.make_cache(spec, 1).to("cuda")
    ctx = gu.context_for(cache)
    raw, zmx = gu.gpu_score(ctx, cache)
    U = cache.n_units
    rows = [cache.unit_rows(u) for u in range(U)]
    N = spec.lens[0]
    Kb = np.stack([r[0] for r in rows]); Pb = np.stack([r[2] for r in rows])
    qm = np.stack([cache.unit_stats(u)[0] for u in range(U)])
    qn = np.stack([cache.unit_stats(u)[1] for u in range(U)])
    RR = np.stack([cache.unit_stats(u)[2] for u in range(U)])
    tt = np.array([cache.t_host[cache.unit_index(u)[1]] for u in range(U)])
    kept_o, nk, zm_o, s_o = oracle.prune_batch(Kb, Pb, np.full(U, N), tt, qm, qn, RR, cache.offsets,
                                               spec.rope_base, spec.budget, spec.layout, want_zmax=True,
                                               want_scores=True)
    # raw scores and max-z of every unit, element by element
    for u in range(U):
        l, b, g = cache.unit_index(u)
        z_o, zmx_o = oracle.zmax(s_o[u])
        assert np.array_equal(zmx_o, zm_o[u])
        orc = {"s": s_o[u], "z": z_o, "zmax": zmx_o}
        gu.check_scores(raw[l, b, g * spec.group:(g + 1) * spec.group], zmx[l, b, g], orc, f"unit {u}")
    st_, code, unit = gu.gpu_prune(ctx, cache)
    assert st_ == tri.TRI_OK, (st_, code, unit)
    for u in range(U):
        l, b, g = cache.unit_index(u)
        out = cache.unit_rows(u)
        kept = gu.kept_from_output(rows[u][2], out[2])
        orc = {"zmax": zm_o[u], "kept": kept_o[u, :nk[u]]}
        gu.check_kept(kept, orc, spec.budget, f"unit {u}")
        gu.check_compacted(rows[u], out, kept, f"unit {u}")
        gu.self_consistent_select(zmx[l, b, g, :N], kept, spec.budget, f"unit {u}")
    ctx.close()


def test_exact_ties_go_to_lower_slots():
    """Identical key rows at different slots are exact ties for the kernel (positions cancel
    in its folded form), so at the threshold it must keep the lowest slots of the boundary
    row. The oracle's literal series un-rotates every key by its own position, which gives
    identical rows fp64 scores that differ in the last bits, so the expectation is built
    from the oracle's ranking of the distinct rows (well separated) plus the tie rule."""
    spec = ts.CacheSpec(name="ties", head_dim=128, group=4, n_kv_heads=1, n_layers=1, batch=1,
                        rope_base=1e6, budget=20, offsets=ts.pow2_offsets(16), positions="from_zero",
                        lens=(64,))
    cache = ts.make_cache(spec, 9).to("cuda")
    # 8 distinct rows, each repeated 8 times (slot i holds row i % 8): ties everywhere
    Kv = cache.K[0, 0, 0]
    Kv[:] = Kv[:8].repeat(8, 1)
    for B in (3, 8, 20, 63):
        c2 = cache.clone()
        rows = c2.unit_rows(0)
        orc = gu.oracle_unit(c2, 0, B, rows=rows)
        # oracle ranking of the distinct rows by their (slot-averaged) max-z
        zrow = np.array([orc["zmax"][r::8].mean() for r in range(8)])
        assert np.all(np.abs(np.subtract.outer(zrow, zrow))[~np.eye(8, dtype=bool)] > 1e-3)
        order = np.argsort(-zrow, kind="stable")
        want = []
        left = B
        for r in order:
            slots = list(range(r, 64, 8))
            want += slots[:left]
            left -= min(left, 8)
            if left == 0:
                break
        want = np.sort(np.array(want))
        ctx = gu.context_for(c2)
        raw, zmx = gu.gpu_score(ctx, c2)
        st, code, unit = gu.gpu_prune(ctx, c2, B)
        assert st == tri.TRI_OK
        out = c2.unit_rows(0)
        kept = gu.kept_from_output(rows[2], out[2])
        gu.check_kept(kept, orc, B)
        gu.self_consistent_select(zmx[0, 0, 0, :64], kept, B)
        assert np.array_equal(kept, want), (B, kept, want)
        gu.check_compacted(rows, out, kept)
        ctx.close()


def test_flat_unit_keeps_first_slots():
    """All keys identical: every z is 0, so the first B slots are kept (and stay in place)."""
    spec = ts.CacheSpec(name="flat", head_dim=64, group=2, n_kv_heads=1, n_layers=1, batch=1,
                        rope_base=1e4, budget=10, offsets=(1, 2, 4), positions="from_zero", lens=(50,))
    cache = ts.make_cache(spec, 2).to("cuda")
    cache.K[0, 0, 0, :50] = cache.K[0, 0, 0, 7]
    rows = cache.unit_rows(0)
    ctx = gu.context_for(cache)
    raw, zmx = gu.gpu_score(ctx, cache)
    assert np.all(zmx[0, 0, 0, :50] == 0.0)
    st, _, _ = gu.gpu_prune(ctx, cache)
    assert st == tri.TRI_OK
    out = cache.unit_rows(0)
    assert np.array_equal(out[2], rows[2][:10])
    ctx.close()


def test_edge_lengths_and_noop():
    """N = 0, 1, B, B + 1 and N < B in one batch: short units untouched, lengths updated."""
    B = 40
    spec = ts.CacheSpec(name="edges", head_dim=128, group=4, n_kv_heads=2, n_layers=1, batch=5,
                        rope_base=1e6, budget=B, offsets=ts.pow2_offsets(16), positions="from_zero",
                        lens=(0, 1, B, B + 1, 25), cap=64)
    cache = ts.make_cache(spec, 4).to("cuda")
    full_parity(cache, label="edges")


def test_layer_chunks_match_one_call():
    """Pruning layer by layer (lens_out NULL, lengths updated at the end) equals one call."""
    spec = _small("qwen3_8b_periodic_36l_3200", n_layers=3, batch=2, n_kv_heads=2, lens=(700, 900),
                  t=(24576, 24576), budget=512)
    a = ts.make_cache(spec, 8).to("cuda")
    b = a.clone()
    ctx = gu.context_for(a)
    ctx.prune(a.K, a.V, a.pos, a.lens, a.t, spec.budget)
    for l in range(spec.n_layers):
        ctx.prune(b.K[l:l + 1], b.V[l:l + 1], b.pos[l:l + 1], b.lens, b.t, spec.budget,
                  lens_out=None, layer_begin=l)
    assert torch.equal(b.lens.cpu(), torch.tensor([700, 900], dtype=torch.int32))
    b.lens.clamp_(max=spec.budget)
    assert _same(a.K, b.K) and _same(a.V, b.V) and _same(a.pos, b.pos)
    assert torch.equal(a.lens, b.lens)
    ctx.close()


def test_device_detected_errors_leave_sequence_untouched():
    spec = ts.CacheSpec(name="bad", head_dim=128, group=4, n_kv_heads=2, n_layers=1, batch=3,
                        rope_base=1e6, budget=30, offsets=ts.pow2_offsets(16), positions="from_zero",
                        lens=(100, 100, 100), cap=128)
    cache = ts.make_cache(spec, 6).to("cuda")
    K0, V0, P0 = _snapshot(cache)
    cache.lens[1] = 129  # above the capacity
    ctx = gu.context_for(cache)
    st = ctx.prune(cache.K, cache.V, cache.pos, cache.lens, cache.t, 30)
    assert st == tri.TRI_OK
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == tri.TRI_DEV_LEN_GT_CAP
    assert cache.unit_index(unit)[1] == 1
    assert _same(cache.K[:, 1], K0[:, 1]) and _same(cache.pos[:, 1], P0[:, 1])
    assert cache.lens_host.tolist() == [30, 129, 30]
    assert ctx.get_error()[0] == tri.TRI_OK  # cleared
    ctx.close()

    # paged: a block-table entry outside the pool
    pspec = _small("qwen3_32b_paged_ragged", n_layers=1, batch=2, lens=(200, 300), budget=64, cap=512)
    pc = ts.make_cache(pspec, 7).to("cuda")
    K0, V0, P0 = _snapshot(pc)
    pc.block_table[0, 1] = pc.n_pages + 5
    ctx = gu.context_for(pc)
    ctx.prune(pc.K, pc.V, pc.pos, pc.lens, pc.t, 64, block_table=pc.block_table)
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == tri.TRI_DEV_BAD_PAGE
    assert pc.lens_host.tolist() == [200, 64]
    for p in range(4):
        if p == 1:
            continue
        pg = int(pc.block_table_host[0, p])
        assert _same(pc.K[:, pg], K0[:, pg]) and _same(pc.pos[:, pg], P0[:, pg])
    ctx.close()


def test_host_validation_with_device():
    spec = ts.WORKLOADS["tiny_d64_n256"]
    cache = ts.make_cache(spec, 0).to("cuda")
    ctx = tri.TriContext(0)
    kv = tri.make_kv(cache.K, cache.V, cache.pos, cache.lens)
    s = torch.cuda.current_stream().cuda_stream
    assert tri.tri_prune(ctx.handle, kv, cache.t.data_ptr(), 64, s) == tri.TRI_ESTATE
    gu_ctx = gu.context_for(cache)
    h = gu_ctx.handle
    assert tri.tri_prune(h, kv, cache.t.data_ptr(), 0, s) == tri.TRI_EINVAL            # budget
    bad = tri.make_kv(cache.K, cache.V, cache.pos, cache.lens); bad.layer_begin = 1
    assert tri.tri_prune(h, bad, cache.t.data_ptr(), 64, s) == tri.TRI_EINVAL          # layer range
    bad = tri.make_kv(cache.K, cache.V, cache.pos, cache.lens); bad.K = cache.K.data_ptr() + 2
    assert tri.tri_prune(h, bad, cache.t.data_ptr(), 64, s) == tri.TRI_EINVAL          # alignment
    host_t = torch.zeros(1, dtype=torch.int32)
    assert tri.tri_prune(h, kv, host_t.data_ptr(), 64, s) == tri.TRI_EINVAL            # host pointer
    bad = tri.make_kv(cache.K, cache.V, cache.pos, cache.lens); bad.cap = 0
    assert tri.tri_prune(h, bad, cache.t.data_ptr(), 64, s) == tri.TRI_EINVAL          # capacity
    q = np.zeros((1, 4, 64), np.float32); r = np.zeros((1, 4, 32), np.float32)
    assert tri.tri_calibrate_load(h, 1, 1, 4, 96, 1e4, 0, q, r, r, [1]) == tri.TRI_EINVAL  # head_dim
    assert tri.tri_calibrate_load(h, 1, 1, 3, 64, 1e4, 0, q, r, r, [1]) == tri.TRI_EINVAL  # group
    qn = q.copy(); qn[0, 0, 0] = np.nan
    assert tri.tri_calibrate_load(h, 1, 1, 4, 64, 1e4, 0, qn, r, r, [1]) == tri.TRI_EINVAL  # non-finite
    assert tri.tri_set_tuning(h, 3, 0) == tri.TRI_EINVAL
    # nothing above launched anything: the cache is unchanged
    assert cache.lens_host.tolist() == [256]
    gu_ctx.close(); ctx.close()


@pytest.mark.parametrize("paged", [False, True])
def test_prune_captured_in_cuda_graph_equals_eager(paged):
    """tri_prune's two launches (the validation kernel, then the fused kernel as its programmatic
    dependent, taking units from a counter the validation zeroes) captured in a CUDA graph and
    replayed give the same cache, bit for bit, as the same call issued directly. Four layers of
    the single-layer decode workload: 512 units, several per cluster."""
    spec = ts.replace(ts.WORKLOADS["qwen3_8b_decode_b16_2176"], n_layers=4,
                      page_size=64 if paged else 0)
    base = ts.make_cache(spec, 41).to("cuda")
    eager, captured = base.clone(), base.clone()
    ctx = gu.context_for(base)
    # the eager call also sizes the context's scratch and caches the launch plan, so the captured
    # call allocates nothing
    assert gu.gpu_prune(ctx, eager)[0] == tri.TRI_OK
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
        ctx.prune(captured.K, captured.V, captured.pos, captured.lens, captured.t, spec.budget,
                  block_table=captured.block_table)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert torch.equal(captured.lens, base.lens)  # capturing ran nothing
    g.replay()
    torch.cuda.synchronize()
    assert ctx.get_error()[0] == tri.TRI_OK
    assert torch.equal(eager.lens, captured.lens)
    assert eager.lens_host.tolist() == [spec.budget] * spec.batch
    assert torch.equal(eager.K.view(torch.int16), captured.K.view(torch.int16))
    assert torch.equal(eager.V.view(torch.int16), captured.V.view(torch.int16))
    assert torch.equal(eager.pos, captured.pos)
    del g
    ctx.close()
