"""tri_calibrate_estimate against the fp64 oracle, through the C ABI.

Seeded query samples (tri_synth.make_queries: per-head centres with spreads from tight to
diffuse, one all-zero band) are reduced on the GPU and by the oracle on the same bits.
Tolerances: the GPU takes |q_f| with one fp32 rounding of re^2 + im^2 and a correctly rounded
fp32 square root (relative error below 1.2e-7 per sample), adds 8 tokens at a time in fp32 (at
most 7 * 2^-24 = 4.2e-7 of the sum of the magnitudes added), adds those partials in fp64, and
rounds the outputs to fp32 once (6e-8). So E|q_f| must agree to 1e-6 relative, the centre to
1e-6 of E|q_f| (it may be near zero; re and im are each bounded by |q_f|), and R (in [0, 1]) to
2e-6 absolute. An all-zero band gives exactly 0.
"""
import numpy as np
import pytest
import torch

import tri_synth as ts
import oracle
from rope_aware_key_tri_b200 import tri

pytestmark = pytest.mark.gpu


def _bits(q):
    return q.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _check(got, want, label):
    qm, qn, R = (x.cpu().numpy().astype(np.float64) for x in got)
    oqm, oqn, oR = want
    assert np.all(np.abs(qn - oqn) <= 1e-6 * oqn + 1e-30), (label, np.max(np.abs(qn - oqn) / (oqn + 1e-30)))
    # the centre may be near zero: measured against the head's largest mean modulus
    assert np.all(np.abs(qm - oqm) <= 1e-6 * np.max(oqn, axis=-1, keepdims=True) + 1e-30), label
    assert np.all(np.abs(R - oR) <= 2e-6), (label, np.max(np.abs(R - oR)))
    assert np.all((R >= 0) & (R <= 1 + 2e-6)), label


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("layout", [tri.TRI_ROPE_HALF, tri.TRI_ROPE_INTERLEAVED])
@pytest.mark.parametrize("L,T,Hq", [(1, 1, 1), (2, 7, 3), (1, 512, 4), (3, 513, 5), (2, 1300, 32)])
def test_matches_oracle(d, layout, L, T, Hq):
    q = ts.make_queries(L, T, Hq, d, seed=L * 1000 + T + Hq + d)
    ctx = tri.TriContext(0)
    got = ctx.calibrate_estimate(q.to("cuda"), layout)
    torch.cuda.synchronize()
    want = oracle.calibrate(_bits(q), layout)
    _check(got, want, f"d={d} layout={layout} L={L} T={T} Hq={Hq}")
    # the all-zero band: exactly zero everywhere
    qn, R = got[1].cpu(), got[2].cpu()
    assert torch.all(qn[:, 0, 0] == 0) and torch.all(R[:, 0, 0] == 0)
    ctx.close()


def test_identical_tokens_give_R_one():
    row = ts.make_queries(1, 1, 2, 128, seed=5)
    q = row.expand(1, 700, 2, 128).contiguous()
    ctx = tri.TriContext(0)
    qm, qn, R = ctx.calibrate_estimate(q.to("cuda"), tri.TRI_ROPE_HALF)
    R = R.cpu().numpy()
    nz = qn.cpu().numpy() > 0
    assert np.all(np.abs(R[nz] - 1.0) <= 2e-7) and np.all(R[~nz] == 0)
    assert torch.equal(qm.cpu(), row[0, 0].float().unsqueeze(0))  # the centre of identical tokens is the token
    ctx.close()


def test_full_size_qwen3_8b_calibration_batch():
    # the pages' calibration batch: about 10K tokens through Qwen3-8B (36 layers, 32 query heads,
    # head_dim 128): 3 GB of bf16 queries; sampled heads against the oracle, and two calls agree
    # bit for bit (fixed summation order)
    L, T, Hq, d = 36, 10240, 32, 128
    q = ts.make_queries(L, T, Hq, d, seed=2024, device="cuda")
    ctx = tri.TriContext(0)
    got = ctx.calibrate_estimate(q, tri.TRI_ROPE_HALF)
    again = ctx.calibrate_estimate(q, tri.TRI_ROPE_HALF)
    torch.cuda.synchronize()
    for a, b in zip(got, again):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    for h in (0, 7, 31):
        sub = q[:, :, h:h + 1, :]
        want = oracle.calibrate(_bits(sub), tri.TRI_ROPE_HALF)
        _check(tuple(x[:, h:h + 1] for x in got), want, f"full size head {h}")
    ctx.close()


def test_estimated_statistics_drive_a_prune():
    # end to end: statistics estimated on the GPU, loaded, and a prune checked against the oracle
    # run with the same (fp32) statistics
    import gpu_util as gu
    spec = ts.replace(ts.WORKLOADS["tiny_d64_n256"], n_kv_heads=2, n_layers=2, batch=2, lens=(256, 180))
    cache = ts.make_cache(spec, 3)
    q = ts.make_queries(spec.n_layers, 300, spec.n_q_heads, spec.head_dim, seed=9)
    ctx = tri.TriContext(0)
    qm, qn, R = (x.cpu().numpy() for x in ctx.calibrate_estimate(q.to("cuda"), spec.layout))
    cache.q_mean, cache.q_norm_mean, cache.R = qm, qn, R
    ctx.calibrate_load(spec.n_layers, spec.n_kv_heads, spec.group, spec.head_dim, spec.rope_base, spec.layout,
                       qm, qn, R, cache.offsets)
    c = cache.to("cuda")
    rows_in = [c.unit_rows(u) for u in range(c.n_units)]
    st, code, unit = gu.gpu_prune(ctx, c)
    assert st == tri.TRI_OK, (st, code, unit)
    for u in range(c.n_units):
        orc = gu.oracle_unit(c, u, spec.budget, rows=rows_in[u])
        kept = gu.kept_from_output(rows_in[u][2], c.unit_rows(u)[2])
        gu.check_kept(kept, orc, spec.budget, f"unit {u}")
    ctx.close()


def test_rejections():
    ctx = tri.TriContext(0)
    q = torch.zeros((1, 4, 2, 96), dtype=torch.bfloat16, device="cuda")
    assert ctx.calibrate_estimate(q, 0, check=False) == tri.TRI_EUNSUPPORTED  # head_dim 96
    qh = torch.zeros((1, 4, 2, 64), dtype=torch.bfloat16)  # host memory
    out = tuple(torch.empty(s, device="cuda") for s in ((1, 2, 64), (1, 2, 32), (1, 2, 32)))
    assert ctx.calibrate_estimate(qh, 0, out=out, check=False) == tri.TRI_EINVAL
    qd = torch.zeros((1 * 4 * 2 * 64 + 1,), dtype=torch.bfloat16, device="cuda")[1:].view(1, 4, 2, 64)
    assert ctx.calibrate_estimate(qd, 0, out=out, check=False) == tri.TRI_EINVAL  # not 16-byte aligned
    assert ctx.get_error()[0] == tri.TRI_OK
    ctx.close()
