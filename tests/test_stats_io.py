"""Calibration statistics on disk (rope_aware_key_tri_b200.stats): round trips through .npz and
.pt, the checks that keep a bad file from reaching a context, and statistics estimated by the
oracle's calibration written and read back unchanged."""
import numpy as np
import pytest
import torch

import oracle
import tri_synth as ts
from rope_aware_key_tri_b200 import stats as S


def _stats(L=2, Hkv=2, G=4, d=64, seed=0, layout=0):
    r = np.random.default_rng(seed)
    Hq = Hkv * G
    qn = r.uniform(0.1, 2.0, (L, Hq, d // 2)).astype(np.float32)
    return S.CalibStats(q_mean=r.normal(size=(L, Hq, d)).astype(np.float32), q_norm_mean=qn,
                        R=r.uniform(0.0, 1.0, (L, Hq, d // 2)).astype(np.float32),
                        offsets=np.array([1, 2, 4, 8], np.int64), n_kv_heads=Hkv, group=G, rope_base=1e4,
                        layout=layout)


def _same(a, b):
    assert a.n_kv_heads == b.n_kv_heads and a.group == b.group and a.layout == b.layout
    assert a.rope_base == b.rope_base
    for k in ("q_mean", "q_norm_mean", "R", "offsets"):
        x, y = getattr(a, k), getattr(b, k)
        assert x.dtype == y.dtype and x.shape == y.shape and np.array_equal(x, y), k


@pytest.mark.parametrize("ext", [".npz", ".pt"])
def test_round_trip(tmp_path, ext):
    s = _stats(layout=1)
    p = str(tmp_path / ("stats" + ext))
    S.save(p, s)
    _same(s, S.load(p))
    assert not (tmp_path / ("stats" + ext + ".tmp")).exists()


@pytest.mark.parametrize("bad", ["head_dim", "group", "heads", "shape", "nan", "R", "base", "layout",
                                 "offsets", "dtype"])
def test_bad_statistics_are_rejected(tmp_path, bad):
    s = _stats()
    if bad == "head_dim":
        s.q_mean = np.zeros((2, 8, 96), np.float32)
    elif bad == "group":
        s.group = 3
    elif bad == "heads":
        s.n_kv_heads = 3
    elif bad == "shape":
        s.R = s.R[:, :, :-1].copy()
    elif bad == "nan":
        s.q_mean[0, 0, 0] = np.nan
    elif bad == "R":
        s.R[0, 0, 0] = 1.5
    elif bad == "base":
        s.rope_base = 0.0
    elif bad == "layout":
        s.layout = 2
    elif bad == "offsets":
        s.offsets = np.zeros(0, np.int64)
    elif bad == "dtype":
        s.q_mean = s.q_mean.astype(np.float64)
    with pytest.raises(S.StatsError):
        S.save(str(tmp_path / "x.npz"), s)


def test_wrong_format_and_missing_fields(tmp_path):
    s = _stats()
    f = S._fields(s)
    p = str(tmp_path / "v2.npz")
    with open(p, "wb") as fh:
        np.savez(fh, **dict(f, format=np.int64(2)))
    with pytest.raises(S.StatsError, match="format"):
        S.load(p)
    p = str(tmp_path / "short.npz")
    with open(p, "wb") as fh:
        np.savez(fh, **{k: v for k, v in f.items() if k != "R"})
    with pytest.raises(S.StatsError, match="missing"):
        S.load(p)


def test_estimated_statistics_survive_the_file(tmp_path):
    """Statistics estimated from query samples by the oracle's calibration, rounded to fp32 as
    the library takes them, come back bit for bit."""
    L, T, Hkv, G, d = 2, 40, 2, 2, 64
    Q = ts.make_queries(L, T, Hkv * G, d, seed=3).view(torch.int16).numpy().view(np.uint16)
    qm, qn, R = oracle.calibrate(Q, 0)
    s = S.from_estimate(qm.astype(np.float32), qn.astype(np.float32), R.astype(np.float32),
                        ts.pow2_offsets(10), Hkv, G, 1e4)
    p = str(tmp_path / "est.npz")
    S.save(p, s)
    _same(s, S.load(p))


@pytest.mark.gpu
def test_context_loaded_from_file_scores_identically(tmp_path):
    """A context fed from a statistics file scores bit for bit like one fed directly."""
    import gpu_util as gu
    from rope_aware_key_tri_b200 import tri
    spec = ts.CacheSpec(name="io", head_dim=128, group=4, n_kv_heads=2, n_layers=2, batch=2, rope_base=1e6,
                        budget=100, offsets=ts.pow2_offsets(16), positions="end_at_t", lens=(300, 211),
                        t=(4000, 900), key_sigma=(0.1, 0.6), cap=320)
    cache = ts.make_cache(spec, 4).to("cuda")
    direct = gu.context_for(cache)
    raw_a, z_a = gu.gpu_score(direct, cache)
    direct.close()
    s = S.CalibStats(q_mean=np.ascontiguousarray(cache.q_mean, np.float32),
                     q_norm_mean=np.ascontiguousarray(cache.q_norm_mean, np.float32),
                     R=np.ascontiguousarray(cache.R, np.float32), offsets=np.asarray(cache.offsets, np.int64),
                     n_kv_heads=spec.n_kv_heads, group=spec.group, rope_base=spec.rope_base, layout=spec.layout)
    p = str(tmp_path / "s.pt")
    S.save(p, s)
    ctx = tri.TriContext(0)
    S.load(p).load_into(ctx)
    raw_b, z_b = gu.gpu_score(ctx, cache)
    ctx.close()
    n = cache.lens_host
    for b in range(spec.batch):
        assert np.array_equal(raw_a[:, b, :, :n[b]], raw_b[:, b, :, :n[b]])
        assert np.array_equal(z_a[:, b, :, :n[b]], z_b[:, b, :, :n[b]])
