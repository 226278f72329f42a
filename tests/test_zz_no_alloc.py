"""tri_prune_noalloc against tri_prune.

Some callers cannot allocate device memory while they run: a serving loop whose device
memory belongs to another allocator, or one that cannot afford the device-wide
synchronisation of a cudaFree. tri_prune_noalloc serves them with fixed, library-held scratch.
Its results must be those of tri_prune within the tolerances of the parity tests: the same
lengths, kept sets equal up to swaps of keys whose max-z lies within 1e-4 of the B-th largest,
and compacted rows that are bit-exact copies of the rows each call kept. Two calls in a row
check that what a previous call left in the fixed scratch does not leak into the next.

This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import tri_synth as ts
import gpu_util as gu
from rope_aware_key_tri_b200 import tri

pytestmark = pytest.mark.gpu


def _kept_slots(rows_in, rows_out):
    return gu.kept_from_output(rows_in[2], rows_out[2])


def test_noalloc_matches_prune_on_two_calls():
    # capacity 65536 at GQA 4: a 1.3 MB score slot per unit, so the fixed 64 MiB holds fewer
    # slots than the resident clusters tri_prune would run; the persistent grid shrinks
    B = 1024
    spec = ts.CacheSpec(name="noalloc", head_dim=128, group=4, n_kv_heads=8, n_layers=2, batch=8,
                        rope_base=1e6, budget=B, offsets=ts.pow2_offsets(16), positions="end_at_t",
                        lens=(3000, 2176, 900, 4000, 1024, 1500, 2600, 3333),
                        t=(9000, 2500, 1000, 30000, 1100, 1600, 2700, 5000), key_sigma=(0.1, 0.6), cap=65536)
    base = ts.make_cache(spec, 31).to("cuda")
    ctx = gu.context_for(base)
    raw, zmx = gu.gpu_score(ctx, base)
    U = base.n_units
    rows_in = [base.unit_rows(u) for u in range(U)]
    lens = base.lens_host.copy()

    ref = base.clone()
    ctx.prune(ref.K, ref.V, ref.pos, ref.lens, ref.t, B)
    assert ctx.get_error()[0] == tri.TRI_OK
    ref_out = [ref.unit_rows(u) for u in range(U)]

    for call in range(2):
        c2 = base.clone()
        ctx.prune_noalloc(c2.K, c2.V, c2.pos, c2.lens, c2.t, B)
        st, code, unit = ctx.get_error()
        assert st == tri.TRI_OK, (call, st, code, unit)
        assert np.array_equal(c2.lens_host, ref.lens_host)
        assert np.array_equal(c2.lens_host, np.minimum(lens, B))
        for u in range(U):
            l, b, g = base.unit_index(u)
            n = int(lens[b])
            out = c2.unit_rows(u)
            kept = _kept_slots(rows_in[u], out)
            kept_ref = _kept_slots(rows_in[u], ref_out[u])
            assert len(kept) == len(kept_ref) == min(n, B)
            z = zmx[l, b, g, :n].astype(np.float64)
            if n > B:
                zb = np.sort(z)[::-1][B - 1]
                diff = np.setxor1d(kept, kept_ref)
                assert np.all(np.abs(z[diff] - zb) <= 1e-4), (call, u, diff)
            gu.check_compacted(rows_in[u], out, kept, f"call {call} unit {u}")
    ctx.close()


def test_noalloc_refusal_does_not_carry_over():
    """The sequence-level verdicts of the allocation-free prune live in the fixed flag array: a
    sequence refused on one call (a cached position not below t) is left untouched, and the
    next call, on a clean copy, prunes it like tri_prune does."""
    spec = ts.CacheSpec(name="noalloc_refuse", head_dim=128, group=4, n_kv_heads=2, n_layers=2, batch=3,
                        rope_base=1e6, budget=100, offsets=ts.pow2_offsets(16), positions="from_zero",
                        lens=(300, 250, 410), key_sigma=(0.1, 0.6), cap=448)
    base = ts.make_cache(spec, 33).to("cuda")
    U = base.n_units
    rows_in = [base.unit_rows(u) for u in range(U)]
    ctx = gu.context_for(base)
    ref = base.clone()
    ctx.prune(ref.K, ref.V, ref.pos, ref.lens, ref.t, spec.budget)
    assert ctx.get_error()[0] == tri.TRI_OK

    bad = base.clone()
    bad.pos[1, 1, 0, spec.lens[1] - 1] = int(bad.t_host[1])  # layer 1, sequence 1, KV head 0
    bad_rows = [bad.unit_rows(u) for u in range(U)]
    ctx.prune_noalloc(bad.K, bad.V, bad.pos, bad.lens, bad.t, spec.budget)
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == tri.TRI_DEV_T_NOT_AFTER_POS
    assert bad.unit_index(unit)[1] == 1
    assert bad.lens_host.tolist() == [100, 250, 100]
    for u in range(U):
        if bad.unit_index(u)[1] == 1:
            out = gu.unit_output_rows(bad, u, spec.lens[1])
            assert all(np.array_equal(x, y) for x, y in zip(out, bad_rows[u])), u

    clean = base.clone()
    ctx.prune_noalloc(clean.K, clean.V, clean.pos, clean.lens, clean.t, spec.budget)
    assert ctx.get_error()[0] == tri.TRI_OK
    assert np.array_equal(clean.lens_host, ref.lens_host)
    for u in range(U):
        out = clean.unit_rows(u)
        kept = _kept_slots(rows_in[u], out)
        assert np.array_equal(kept, _kept_slots(rows_in[u], ref.unit_rows(u))), u
        gu.check_compacted(rows_in[u], out, kept, f"unit {u}")
    ctx.close()


def test_noalloc_limits_are_rejected_without_launch():
    # a unit capacity of 2^21 slots: no launch shape keeps its keep mask on chip, so both entry
    # points refuse it (for every capacity tri_prune accepts, one score slot stays far below the
    # fixed 64 MiB); nothing is launched
    spec = ts.CacheSpec(name="noalloc_big", head_dim=64, group=8, n_kv_heads=1, n_layers=1, batch=1,
                        rope_base=1e4, budget=16, offsets=(1, 2), positions="from_zero", lens=(64,),
                        cap=1 << 21)
    c = ts.make_cache(spec, 5).to("cuda")
    ctx = gu.context_for(c)
    K0 = c.K[0, 0, 0, :64].clone()
    st = ctx.prune_noalloc(c.K, c.V, c.pos, c.lens, c.t, 16, check=False)
    assert st == tri.TRI_EUNSUPPORTED
    assert "capacity" in tri.tri_last_error(ctx.handle)
    assert ctx.prune(c.K, c.V, c.pos, c.lens, c.t, 16, check=False) == tri.TRI_EUNSUPPORTED
    torch.cuda.synchronize()
    assert torch.equal(c.K[0, 0, 0, :64].view(torch.int16), K0.view(torch.int16))
    assert c.lens_host.tolist() == [64]
    ctx.close()

    # more sequences than the fixed flag array holds: refused with a clear message
    spec2 = ts.CacheSpec(name="noalloc_batch", head_dim=64, group=1, n_kv_heads=1, n_layers=1, batch=16385,
                         rope_base=1e4, budget=4, offsets=(1,), positions="from_zero", lens=(0,) * 16385, cap=16)
    c2 = ts.make_cache(spec2, 6).to("cuda")
    ctx2 = gu.context_for(c2)
    st = ctx2.prune_noalloc(c2.K, c2.V, c2.pos, c2.lens, c2.t, 4, check=False)
    assert st == tri.TRI_EUNSUPPORTED
    assert "16384" in tri.tri_last_error(ctx2.handle)
    # the allocating entry point takes the same batch
    assert ctx2.prune(c2.K, c2.V, c2.pos, c2.lens, c2.t, 4, check=False) == tri.TRI_OK
    assert ctx2.get_error()[0] == tri.TRI_OK
    ctx2.close()
