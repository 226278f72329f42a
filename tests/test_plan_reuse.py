"""One context across call shapes.

The library keeps the last launch plan and reuses it while the call shape (unit capacity,
unit count, tuning) repeats. A context that alternates between shapes, and between tunings,
must plan each call for its own shape: every prune below is checked against the fp64 oracle.
"""
import numpy as np
import pytest

import tri_synth as ts
import gpu_util as gu
from rope_aware_key_tri_b200 import tri

pytestmark = pytest.mark.gpu

BASE = ts.CacheSpec(name="reuse", head_dim=128, group=4, n_kv_heads=2, n_layers=2, batch=2,
                    rope_base=1e6, budget=96, offsets=ts.pow2_offsets(12), positions="end_at_t",
                    lens=(700, 260), t=(900, 300), key_sigma=(0.2, 0.5))

SHAPES = [
    BASE,
    ts.replace(BASE, batch=3, lens=(2100, 97, 1500), t=(2200, 97, 1600)),   # more units, larger capacity
    BASE,                                                                    # back to the first shape
    ts.replace(BASE, lens=(5000, 4000), t=(5000, 4100), budget=1024),         # several compaction rounds
]


def _prune_and_check(ctx, spec, seed, label):
    cache = ts.make_cache(spec, seed).to("cuda")
    B = spec.budget
    rows_in = [cache.unit_rows(u) for u in range(cache.n_units)]
    lens = cache.lens_host.copy()
    st, code, unit = gu.gpu_prune(ctx, cache, B)
    assert st == tri.TRI_OK, (label, st, code, unit)
    assert np.array_equal(cache.lens_host, np.minimum(lens, B)), label
    for u in range(cache.n_units):
        orc = gu.oracle_unit(cache, u, B, rows=rows_in[u])
        out = cache.unit_rows(u)
        kept = gu.kept_from_output(rows_in[u][2], out[2])
        gu.check_kept(kept, orc, B, f"{label} unit {u}")
        gu.check_compacted(rows_in[u], out, kept, f"{label} unit {u}")


def test_one_context_many_shapes_and_tunings():
    # the calibration statistics depend only on the model shape and the seed, so every cache
    # below shares them with the context
    first = ts.make_cache(SHAPES[0], 77)
    ctx = gu.context_for(first)
    for i, spec in enumerate(SHAPES):
        _prune_and_check(ctx, spec, 77, f"shape {i}")
    for cs, nb in ((1, 2), (4, 1), (0, 0), (2, 3)):
        ctx.set_tuning(cs, nb)
        _prune_and_check(ctx, SHAPES[1], 77, f"tuning {cs}:{nb}")
    ctx.close()
