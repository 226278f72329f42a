"""Device-detected failures, through the C ABI, in both offset modes.

Sequence-level problems (here: a cached position that is not below t) are decided by the
validation kernel before any unit is touched: the whole sequence stays as it was and keeps its
length. Unit-level failures are made on purpose with the library's test hook, which withholds
one key copy so that the bounded wait for it runs out after a few tries (no copy is left in
flight, nothing waits without bound): only the affected units stay uncompacted, the other units
are pruned as the oracle says, every length becomes min(len, B), and the affected units are
listed by tri_get_failed_units.
"""
import numpy as np
import pytest
import torch

import tri_synth as ts
import gpu_util as gu
from rope_aware_key_tri_b200 import tri

pytestmark = pytest.mark.gpu


def _same(a, b):
    if a.dtype == torch.bfloat16:
        a, b = a.view(torch.int16), b.view(torch.int16)
    return torch.equal(a, b)


def _check_pruned_unit(cache, u, rows_in, B, combine, label):
    orc = gu.oracle_unit(cache, u, B, rows=rows_in, combine=combine)
    n = len(rows_in[2])
    out = gu.unit_output_rows(cache, u, min(n, B))
    kept = gu.kept_from_output(rows_in[2], out[2])
    gu.check_kept(kept, orc, B, label)
    gu.check_compacted(rows_in, out, kept, label)


def _check_untouched_unit(cache, u, rows_in, label):
    n = len(rows_in[2])
    out = gu.unit_output_rows(cache, u, n)
    for a, b, what in zip(out, rows_in, ("K", "V", "pos")):
        assert np.array_equal(a, b), f"{label}: {what} of a unit that must stay untouched changed"


@pytest.mark.parametrize("combine", ["mean", "max"])
@pytest.mark.parametrize("paged", [False, True], ids=["dense", "paged"])
def test_position_not_below_t_refuses_the_sequence(combine, paged):
    if paged:
        spec = ts.replace(ts.WORKLOADS["qwen3_32b_paged_ragged"], n_layers=2, batch=3, lens=(300, 250, 410),
                          budget=100, cap=512)
    else:
        spec = ts.CacheSpec(name="tpos", head_dim=128, group=4, n_kv_heads=2, n_layers=2, batch=3,
                            rope_base=1e6, budget=100, offsets=ts.pow2_offsets(16), positions="from_zero",
                            lens=(300, 250, 410), key_sigma=(0.1, 0.6), cap=448)
    cache = ts.make_cache(spec, 21).to("cuda")
    U = cache.n_units
    # one unit of sequence 1 (layer 1, KV head 1) gets a last position equal to t
    bad_u = (1 * spec.batch + 1) * spec.n_kv_heads + 1
    l, b, g = cache.unit_index(bad_u)
    n = spec.lens[1]
    t1 = int(cache.t_host[1])
    if paged:
        ps = spec.page_size
        pg = int(cache.block_table_host[1, (n - 1) // ps])
        cache.pos[l, pg, g, (n - 1) % ps] = t1
    else:
        cache.pos[l, b, g, n - 1] = t1
    rows = [cache.unit_rows(u) for u in range(U)]
    ctx = gu.context_for(cache, combine=combine)
    st, code, unit = gu.gpu_prune(ctx, cache, spec.budget)
    assert st == tri.TRI_EDEVICE and code == tri.TRI_DEV_T_NOT_AFTER_POS, (st, code)
    assert unit == bad_u
    assert cache.lens_host.tolist() == [100, 250, 100]
    for u in range(U):
        lab = f"{combine} unit {u}"
        if cache.unit_index(u)[1] == 1:
            _check_untouched_unit(cache, u, rows[u], lab)
        else:
            _check_pruned_unit(cache, u, rows[u], spec.budget, combine, lab)
    assert ctx.failed_units() == (0, [])
    ctx.close()


def _fault_case():
    spec = ts.CacheSpec(name="fault", head_dim=128, group=4, n_kv_heads=4, n_layers=2, batch=8,
                        rope_base=1e6, budget=100, offsets=ts.pow2_offsets(16), positions="from_zero",
                        lens=(300, 120, 260, 300, 90, 300, 230, 300), key_sigma=(0.1, 0.6), cap=320)
    return spec, ts.make_cache(spec, 23).to("cuda")


@pytest.mark.parametrize("combine", ["mean", "max"])
def test_withheld_copy_times_out_and_leaves_units_uncompacted(combine):
    spec, cache = _fault_case()
    U = cache.n_units
    rows = [cache.unit_rows(u) for u in range(U)]
    lens0 = cache.lens_host.copy()
    victim = 5  # layer 0, sequence 1, KV head 1 (120 keys, more than the budget)
    assert lens0[cache.unit_index(victim)[1]] > spec.budget
    ctx = gu.context_for(cache, combine=combine)
    if combine == "mean":
        ctx.set_tuning(cluster_size=16)  # few clusters: the failing one has later units to refuse
    ctx.set_test_fault(victim, wait_tries=4)
    st, code, unit = gu.gpu_prune(ctx, cache, spec.budget)
    assert st == tri.TRI_EDEVICE and code == tri.TRI_DEV_TIMEOUT, (st, code, unit)
    n_failed, failed = ctx.failed_units()
    assert n_failed == len(failed) and victim in failed
    failed = sorted(set(failed))
    if combine == "mean":
        # units are handed out dynamically: the cluster whose wait ran out refuses the unit it had
        # already taken next (when that one needs pruning) and takes no more
        assert len(failed) <= 2, failed
        assert all(lens0[cache.unit_index(u)[1]] > spec.budget for u in failed), failed
    else:
        # the tensor-core scoring kernel refuses the units of the tile range it abandoned
        if len(failed) > 1:
            c = int(np.gcd.reduce(np.diff(failed)))
            want = [u for u in range(victim, U, c)
                    if lens0[cache.unit_index(u)[1]] > spec.budget]
            assert failed == want, (failed, want)
    # every sequence gets min(len, B); listed units keep their original rows, the others are pruned
    assert cache.lens_host.tolist() == np.minimum(lens0, spec.budget).tolist()
    for u in range(U):
        lab = f"{combine} unit {u}"
        if u in failed:
            _check_untouched_unit(cache, u, rows[u], lab)
        else:
            _check_pruned_unit(cache, u, rows[u], spec.budget, combine, lab)
    # read and cleared
    assert ctx.get_error()[0] == tri.TRI_OK
    assert ctx.failed_units() == (0, [])

    # hook off: the same context prunes a fresh copy completely
    ctx.set_test_fault(-1, 0)
    spec, fresh = _fault_case()
    st, code, unit = gu.gpu_prune(ctx, fresh, spec.budget)
    assert st == tri.TRI_OK, (st, code, unit)
    for u in range(U):
        _check_pruned_unit(fresh, u, rows[u], spec.budget, combine, f"{combine} fresh unit {u}")
    assert ctx.failed_units() == (0, [])
    ctx.close()
