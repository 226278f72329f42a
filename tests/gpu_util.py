"""Helpers for the GPU parity tests: run the CUDA path through the C-ABI binding and compare
its results with the fp64 oracle on the same seeded inputs.

Tolerances (all stated by the pass's contract):
  * raw scores: |s_gpu - s_oracle| <= 1e-4 * max_i |s_oracle,h(i)| per query head;
  * kept sets: equal, except that keys whose oracle max-z lies within 1e-4 of the
    B-th largest oracle max-z may be swapped;
  * compacted K, V and positions: bit-exact copies of the rows the GPU kept.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from rope_aware_key_tri_b200 import tri

SCORE_RTOL = 1e-4
Z_TIE = 1e-4


def context_for(cache, cluster_size=0, buffers=0, combine="mean", engine="auto"):
    s = cache.spec
    ctx = tri.TriContext(0)
    ctx.calibrate_load(s.n_layers, s.n_kv_heads, s.group, s.head_dim, s.rope_base, s.layout,
                       cache.q_mean, cache.q_norm_mean, cache.R, cache.offsets)
    if cluster_size or buffers:
        ctx.set_tuning(cluster_size, buffers)
    if combine != "mean":
        ctx.set_offset_combine(combine)
    if engine != "auto":
        ctx.set_score_engine(engine)
    return ctx


def gpu_score(ctx, cache, layer_begin=0, n_layers=None):
    """(raw [nl][batch][Hq][cap_u], zmax [nl][batch][Hkv][cap_u]) as numpy, via tri_score."""
    s = cache.spec
    nl = s.n_layers if n_layers is None else n_layers
    K = cache.K[layer_begin:layer_begin + nl]
    raw = torch.full((nl, s.batch, s.n_q_heads, cache.cap), float("nan"), device="cuda")
    zmx = torch.full((nl, s.batch, s.n_kv_heads, cache.cap), float("nan"), device="cuda")
    ctx.score(K, cache.lens, cache.t, raw=raw, zmax=zmx, block_table=cache.block_table,
              layer_begin=layer_begin)
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_OK, (st, code, unit)
    return raw.cpu().numpy(), zmx.cpu().numpy()


def gpu_prune(ctx, cache, budget=None, lens_out="inplace"):
    s = cache.spec
    B = s.budget if budget is None else budget
    lo = cache.lens if isinstance(lens_out, str) else lens_out
    ctx.prune(cache.K, cache.V, cache.pos, cache.lens, cache.t, B, lens_out=lo,
              block_table=cache.block_table)
    return ctx.get_error()


def oracle_unit(cache, u, B, rows=None, combine="mean"):
    s = cache.spec
    k, v, p = rows if rows is not None else cache.unit_rows(u)
    qm, qn, R = cache.unit_stats(u)
    _, b, _ = cache.unit_index(u)
    return oracle.prune_unit(k, v, p, int(cache.t_host[b]), qm, qn, R, cache.offsets, s.rope_base, B,
                             s.layout, combine=combine)


def zmax_bound(s_err, s_orc, z_orc):
    """Largest |zmax_gpu - zmax_oracle| that score errors of at most s_err[h] per head allow.

    With |s_gpu - s| <= e per key, the mean moves by at most e and the population std by at
    most 2e (the centred vectors differ by at most 2e per key), so
    |z_gpu - z| <= (2 + 2|z|) e / (sigma - 2e); zmax, a max over the heads, moves by at most
    the largest head bound. Added: the fp32 evaluation of (s - mu) / sigma and the max
    (a few ulps of |z|). A flat head (sigma = 0) has z = 0 on both sides."""
    G, n = s_orc.shape
    bound = 0.0
    for h in range(G):
        sig = s_orc[h].std()
        if not (s_orc[h].max() > s_orc[h].min()):
            continue
        # the kernel's mean is rounded to fp32 before the subtraction: an error of up to
        # 2^-24 |mu| on top of the score's own
        e = float(s_err[h]) + 2.0 ** -24 * abs(float(s_orc[h].mean()))
        if sig <= 2 * e:
            return np.inf
        bound = max(bound, (2.0 + 2.0 * np.abs(z_orc[h]).max()) * e / (sig - 2 * e))
    return bound + 4e-7 * (1.0 + np.abs(z_orc).max())


def check_scores(raw_u, zmax_u, orc, label=""):
    """raw_u [G][n] and zmax_u [n] from the GPU against the oracle's s and zmax."""
    s = orc["s"]
    G, n = s.shape
    errs = np.zeros(G)
    for h in range(G):
        scale = np.abs(s[h]).max() if n else 0.0
        err = np.abs(raw_u[h, :n].astype(np.float64) - s[h]).max() if n else 0.0
        assert err <= SCORE_RTOL * scale + 1e-30, f"{label} head {h}: score error {err:.3e} vs scale {scale:.3e}"
        errs[h] = err
    if n:
        zerr = np.abs(zmax_u[:n].astype(np.float64) - orc["zmax"]).max()
        zb = zmax_bound(errs, s, orc["z"])
        assert zerr <= zb, f"{label}: zmax error {zerr:.3e} above the bound {zb:.3e} the score errors allow"


def kept_from_output(in_pos, out_pos):
    """Source slots of the GPU's kept rows, recovered from the (unique) positions."""
    idx = np.searchsorted(in_pos, out_pos)
    assert np.all(idx < len(in_pos)) and np.array_equal(in_pos[idx], out_pos), "output position not in input"
    return idx


def check_kept(gpu_kept, orc, B, label=""):
    n = orc["zmax"].shape[0]
    M = min(n, B)
    assert len(gpu_kept) == M, f"{label}: kept {len(gpu_kept)} != {M}"
    assert np.all(np.diff(gpu_kept) > 0), f"{label}: kept slots not strictly ascending"
    if n <= B:
        assert np.array_equal(gpu_kept, np.arange(n))
        return 0
    zb = np.sort(orc["zmax"])[::-1][B - 1]
    diff = np.setxor1d(gpu_kept, orc["kept"])
    bad = diff[np.abs(orc["zmax"][diff] - zb) > Z_TIE]
    assert len(bad) == 0, f"{label}: {len(bad)} kept-set differences beyond the threshold tie band"
    return len(diff)


def check_compacted(in_rows, out_rows, gpu_kept, label=""):
    k, v, p = in_rows
    ko, vo, po = out_rows
    assert np.array_equal(ko, k[gpu_kept]), f"{label}: K rows differ"
    assert np.array_equal(vo, v[gpu_kept]), f"{label}: V rows differ"
    assert np.array_equal(po, p[gpu_kept]), f"{label}: positions differ"


def self_consistent_select(zmax_gpu, gpu_kept, B, label=""):
    """The GPU's kept set is exactly the top-B of its own max-z, ties to the lower slot."""
    n = zmax_gpu.shape[0]
    if n <= B:
        return
    order = np.lexsort((np.arange(n), -zmax_gpu.astype(np.float64)))
    want = np.sort(order[:B])
    assert np.array_equal(want, gpu_kept), f"{label}: select differs from top-B of the GPU's own max-z"


def unit_output_rows(cache, u, M):
    """First M rows of unit u after pruning (host numpy)."""
    s = cache.spec
    saved = cache.lens
    l, b, g = cache.unit_index(u)
    cache.lens = cache.lens.clone()
    cache.lens[b] = M
    try:
        return cache.unit_rows(u)
    finally:
        cache.lens = saved


def row_hashes(x: torch.Tensor, coeff: torch.Tensor) -> torch.Tensor:
    """64-bit (wrapping) hash of each row of an int16 view [..., d]."""
    return (x.to(torch.int64) * coeff).sum(-1)
