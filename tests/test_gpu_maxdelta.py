"""GPU parity of the max-over-offsets mode (tri_set_offset_combine(TRI_OFFSETS_MAX)): the
tensor-core scoring kernel plus the fused z-score / select / compaction, through the C ABI,
against the oracle's max mode (trigonometric term = max over delta of the literal series, as
in the TriAttention deep-dive page, §3.3 and the scoring code of its §4.2).

Tolerances are those of the mean mode: raw scores within 1e-4 of each head's largest |s|,
kept sets equal up to threshold ties, compacted rows bit-exact.
"""
import numpy as np
import pytest
import torch

import tri_synth as ts
import gpu_util as gu
from rope_aware_key_tri_b200 import tri
from test_gpu_parity import _same, _small, _snapshot, full_parity

pytestmark = pytest.mark.gpu


def _score_check(cache, combine="max"):
    s = cache.spec
    ctx = gu.context_for(cache, combine=combine)
    raw, zmx = gu.gpu_score(ctx, cache)
    for u in range(cache.n_units):
        l, b, g = cache.unit_index(u)
        orc = gu.oracle_unit(cache, u, s.budget, combine=combine)
        gu.check_scores(raw[l, b, g * s.group:(g + 1) * s.group], zmx[l, b, g], orc,
                        f"{combine} unit {u} (N={cache.lens_host[b]})")
    ctx.close()
    return raw, zmx


@pytest.mark.parametrize("layout", [ts.HALF, ts.INTERLEAVED], ids=["half", "interleaved"])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_max_scores_shapes(head_dim, group, layout):
    """Raw scores and max-z of every unit; lengths 301 and 517 span several 128-key tiles and
    end in a ragged tile."""
    spec = ts.CacheSpec(name="mx", head_dim=head_dim, group=group, n_kv_heads=2, n_layers=2, batch=2,
                        rope_base=1e6 if head_dim == 128 else 1e4, budget=200,
                        offsets=ts.pow2_offsets(16), positions="end_at_t", lens=(301, 517),
                        t=(9000, 700), key_sigma=(0.1, 0.6), layout=layout, cap=640)
    cache = ts.make_cache(spec, 101 + head_dim + group + 7 * layout).to("cuda")
    _score_check(cache)


@pytest.mark.parametrize("group", [4, 8])
def test_max_prune_dense(group):
    spec = ts.CacheSpec(name="mxp", head_dim=128, group=group, n_kv_heads=2, n_layers=2, batch=3,
                        rope_base=1e6, budget=333, offsets=ts.pow2_offsets(16), positions="periodic",
                        lens=(1501, 1000, 334), t=(20000, 5000, 900), key_sigma=(0.1, 0.6), recent=128)
    cache = ts.make_cache(spec, 17 + group).to("cuda")
    full_parity(cache, label=f"max G{group}", combine="max")


@pytest.mark.parametrize("page_size", [16, 64])
def test_max_prune_paged(page_size):
    spec = ts.replace(ts.WORKLOADS["qwen3_32b_paged_ragged"], n_layers=2, batch=3, lens=(700, 129, 513),
                      page_size=page_size, budget=128, cap=1024)
    cache = ts.make_cache(spec, 23).to("cuda")
    full_parity(cache, label=f"max paged{page_size}", combine="max")


def test_max_prune_small_offset_set_d64():
    """The small d = 64 workload (offsets 2^0..2^10, 11 per head) end to end."""
    cache = ts.make_cache(ts.WORKLOADS["tiny_d64_n256"], 0).to("cuda")
    full_parity(cache, label="max tiny", combine="max")


def test_one_offset_max_equals_mean():
    """With a single offset the maximum and the mean are the same number: the two GPU modes
    (tensor-core contraction vs folded fp32 dot product) must agree within the score tolerance,
    and both with the oracle."""
    spec = ts.CacheSpec(name="one", head_dim=128, group=4, n_kv_heads=2, n_layers=1, batch=2,
                        rope_base=1e6, budget=100, offsets=(7,), positions="end_at_t", lens=(260, 389),
                        t=(5000, 12000), key_sigma=(0.1, 0.6), cap=512)
    cache = ts.make_cache(spec, 5).to("cuda")
    raw_max, _ = _score_check(cache, "max")
    raw_mean, _ = _score_check(cache, "mean")
    for u in range(cache.n_units):
        l, b, g = cache.unit_index(u)
        n = cache.lens_host[b]
        a = raw_max[l, b, g * 4:(g + 1) * 4, :n].astype(np.float64)
        m = raw_mean[l, b, g * 4:(g + 1) * 4, :n].astype(np.float64)
        scale = np.abs(m).max(axis=1, keepdims=True)
        assert (np.abs(a - m) <= 2e-4 * scale).all()


def test_max_mode_switches_back():
    """Switching the context back to the mean gives the mean-mode results again."""
    spec = ts.CacheSpec(name="sw", head_dim=64, group=2, n_kv_heads=1, n_layers=1, batch=1,
                        rope_base=1e4, budget=50, offsets=ts.pow2_offsets(10), positions="end_at_t",
                        lens=(200,), t=(300,), key_sigma=(0.2, 0.4), cap=256)
    cache = ts.make_cache(spec, 9).to("cuda")
    ctx = gu.context_for(cache, combine="max")
    ctx.set_offset_combine("mean")
    raw, zmx = gu.gpu_score(ctx, cache)
    orc = gu.oracle_unit(cache, 0, spec.budget)
    gu.check_scores(raw[0, 0, 0:2], zmx[0, 0, 0], orc, "mean after max")
    ctx.close()


def test_max_noalloc_refused():
    spec = ts.WORKLOADS["tiny_d64_n256"]
    cache = ts.make_cache(spec, 0).to("cuda")
    ctx = gu.context_for(cache, combine="max")
    with pytest.raises(tri.TriError) as e:
        ctx.prune_noalloc(cache.K, cache.V, cache.pos, cache.lens, cache.t, spec.budget,
                          block_table=cache.block_table)
    assert e.value.status == tri.TRI_EUNSUPPORTED
    ctx.close()


def test_max_edge_lengths_and_noop():
    """N = 0, 1, B, B + 1 and N < B in one batch: only the unit above the budget is scored and
    pruned; the others keep their rows and lengths."""
    B = 40
    spec = ts.CacheSpec(name="mx_edges", head_dim=128, group=4, n_kv_heads=2, n_layers=1, batch=5,
                        rope_base=1e6, budget=B, offsets=ts.pow2_offsets(16), positions="from_zero",
                        lens=(0, 1, B, B + 1, 25), cap=64)
    cache = ts.make_cache(spec, 4).to("cuda")
    full_parity(cache, label="max edges", combine="max")


def test_max_layer_chunks_match_one_call():
    """Layer by layer (lens_out NULL, lengths updated at the end) equals one call, in max mode."""
    spec = _small("qwen3_8b_periodic_36l_3200", n_layers=3, batch=2, n_kv_heads=2, lens=(700, 900),
                  t=(24576, 24576), budget=512)
    a = ts.make_cache(spec, 8).to("cuda")
    b = a.clone()
    ctx = gu.context_for(a, combine="max")
    ctx.prune(a.K, a.V, a.pos, a.lens, a.t, spec.budget)
    for l in range(spec.n_layers):
        ctx.prune(b.K[l:l + 1], b.V[l:l + 1], b.pos[l:l + 1], b.lens, b.t, spec.budget,
                  lens_out=None, layer_begin=l)
    assert torch.equal(b.lens.cpu(), torch.tensor([700, 900], dtype=torch.int32))
    b.lens.clamp_(max=spec.budget)
    assert _same(a.K, b.K) and _same(a.V, b.V) and _same(a.pos, b.pos)
    assert torch.equal(a.lens, b.lens)
    ctx.close()


def test_max_device_detected_errors_leave_sequence_untouched():
    spec = ts.CacheSpec(name="mx_bad", head_dim=128, group=4, n_kv_heads=2, n_layers=1, batch=3,
                        rope_base=1e6, budget=30, offsets=ts.pow2_offsets(16), positions="from_zero",
                        lens=(100, 100, 100), cap=128)
    cache = ts.make_cache(spec, 6).to("cuda")
    K0, V0, P0 = _snapshot(cache)
    cache.lens[1] = 129  # above the capacity
    ctx = gu.context_for(cache, combine="max")
    ctx.prune(cache.K, cache.V, cache.pos, cache.lens, cache.t, 30)
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == tri.TRI_DEV_LEN_GT_CAP
    assert cache.unit_index(unit)[1] == 1
    assert _same(cache.K[:, 1], K0[:, 1]) and _same(cache.pos[:, 1], P0[:, 1])
    assert cache.lens_host.tolist() == [30, 129, 30]
    ctx.close()

    # paged: a block-table entry outside the pool (the scoring kernel loads none of it)
    pspec = _small("qwen3_32b_paged_ragged", n_layers=1, batch=2, lens=(200, 300), budget=64, cap=512)
    pc = ts.make_cache(pspec, 7).to("cuda")
    K0, V0, P0 = _snapshot(pc)
    pc.block_table[0, 1] = pc.n_pages + 5
    ctx = gu.context_for(pc, combine="max")
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


@pytest.mark.parametrize("page_size", [32, 48])
def test_max_prune_paged_odd_pages(page_size):
    """Pages of 32 and 48 slots: the key tiles are loaded in boxes of 32 and 16 rows."""
    spec = ts.replace(ts.WORKLOADS["qwen3_32b_paged_ragged"], n_layers=1, batch=2, lens=(400, 257),
                      page_size=page_size, budget=100, cap=480)
    cache = ts.make_cache(spec, 31).to("cuda")
    full_parity(cache, label=f"max paged{page_size}", combine="max")
