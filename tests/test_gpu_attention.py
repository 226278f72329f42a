"""Decode attention over the (pruned) cache on the GPU, through the C ABI, against the fp64
oracle (tri_oracle_decode_attention) element by element.

Tolerance, derived from the kernel's arithmetic (fp32 throughout, bf16 inputs exact):
  * a logit (scaled into the log2 domain) is a sum of d products, each rounded once, plus the
    rounding of the scaled query: |error| <= (d + 2) 2^-24 max_j sum_i |q_i k_ji| qscale;
  * a softmax weight 2^(x - m) then moves by a factor of at most 2^(2 e) (the logit and the
    running max), plus 4 ulps for the hardware exp2 and the rescales;
  * the weighted sum of M values and the normaliser accumulate in fp32: (M + 8) 2^-24 relative;
so |out - oracle| <= (2 ln2 e + 2^-20 + (M + 8) 2^-24) max_j |v_j| (first order), per unit and
query head. A sequence of length 0 gets zeros.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import tri_synth as ts
import gpu_util as gu
from rope_aware_key_tri_b200 import tri

pytestmark = pytest.mark.gpu


def _bf16_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _queries(spec, seed, device="cuda"):
    g = torch.Generator().manual_seed(seed)
    q = 2.0 * torch.randn((spec.n_layers, spec.batch, spec.n_q_heads, spec.head_dim), generator=g)
    return q.to(torch.bfloat16).to(device)


def _bound(qb, Kb, Vb):
    d = qb.shape[1]
    qscale = math.log2(math.e) / math.sqrt(d)
    qv = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    kv = (Kb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    vv = (Vb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    M = Kb.shape[0]
    e = (d + 2) * 2.0 ** -24 * (np.abs(qv) @ np.abs(kv).T).max() * qscale
    return (2 * math.log(2) * e + 2.0 ** -20 + (M + 8) * 2.0 ** -24) * np.abs(vv).max()


def check_attention(cache, q, out, lens=None, label=""):
    s = cache.spec
    lens = cache.lens_host if lens is None else lens
    o = out.cpu().numpy()
    qb_all = _bf16_bits(q)
    worst = 0.0
    for u in range(cache.n_units):
        l, b, g = cache.unit_index(u)
        n = int(lens[b])
        got = o[l, b, g * s.group:(g + 1) * s.group]
        if n == 0:
            assert np.all(got == 0.0), f"{label} unit {u}: empty sequence must give zeros"
            continue
        k, v, _ = gu.unit_output_rows(cache, u, n)
        qb = qb_all[l, b, g * s.group:(g + 1) * s.group]
        want = oracle.decode_attention(qb, k, v)
        err = np.abs(got.astype(np.float64) - want).max()
        tol = _bound(qb, k, v)
        assert err <= tol, f"{label} unit {u} (n={n}): error {err:.3e} above the bound {tol:.3e}"
        worst = max(worst, err / tol)
    return worst


@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_attention_shapes_dense(head_dim, group):
    spec = ts.CacheSpec(name="att", head_dim=head_dim, group=group, n_kv_heads=2, n_layers=2, batch=7,
                        rope_base=1e6, budget=64, offsets=(1,), positions="from_zero",
                        lens=(0, 1, 15, 16, 17, 100, 333), key_sigma=(0.1, 0.6), cap=352)
    cache = ts.make_cache(spec, 40 + head_dim + group).to("cuda")
    q = _queries(spec, 41 + group)
    ctx = gu.context_for(cache)
    out = torch.full(q.shape, float("nan"), device="cuda")
    ctx.decode_attention(cache.K, cache.V, cache.lens, q, out=out)
    assert ctx.get_error()[0] == tri.TRI_OK
    check_attention(cache, q, out, label=f"d{head_dim} G{group}")
    ctx.close()


@pytest.mark.parametrize("page_size", [16, 64])
def test_attention_paged_permuted(page_size):
    spec = ts.replace(ts.WORKLOADS["qwen3_32b_paged_ragged"], n_layers=2, batch=4, lens=(700, 0, 129, 513),
                      page_size=page_size, budget=128, cap=1024)
    cache = ts.make_cache(spec, 42).to("cuda")
    q = _queries(spec, 43)
    ctx = gu.context_for(cache)
    out = ctx.decode_attention(cache.K, cache.V, cache.lens, q, block_table=cache.block_table)
    assert ctx.get_error()[0] == tri.TRI_OK
    check_attention(cache, q, out, label=f"paged{page_size}")
    ctx.close()


def test_attention_split_into_chunks():
    """Two long units: each is split over many CTAs whose partials the combine launch merges."""
    spec = ts.CacheSpec(name="att_long", head_dim=128, group=4, n_kv_heads=1, n_layers=1, batch=2,
                        rope_base=1e6, budget=64, offsets=(1,), positions="from_zero",
                        lens=(9000, 4099), key_sigma=(0.1, 0.6))
    cache = ts.make_cache(spec, 44).to("cuda")
    q = _queries(spec, 45)
    ctx = gu.context_for(cache)
    out = ctx.decode_attention(cache.K, cache.V, cache.lens, q)
    assert ctx.get_error()[0] == tri.TRI_OK
    check_attention(cache, q, out, label="split")
    ctx.close()


@pytest.mark.parametrize("name", ["qwen3_8b_decode_b16_2176", "qwen3_32b_paged_ragged"])
def test_attention_after_prune(name):
    """Prune with tri_prune, then attend over the kept rows (non-contiguous positions)."""
    if name == "qwen3_32b_paged_ragged":
        spec = ts.replace(ts.WORKLOADS[name], n_layers=2, batch=4, lens=(2500, 2176, 3000, 900), cap=3072)
    else:
        spec = ts.replace(ts.WORKLOADS[name], batch=4, lens=(2176,) * 4)
    cache = ts.make_cache(spec, 46).to("cuda")
    ctx = gu.context_for(cache)
    st, code, unit = gu.gpu_prune(ctx, cache, spec.budget)
    assert st == tri.TRI_OK, (st, code, unit)
    assert np.all(cache.lens_host <= spec.budget)
    q = _queries(spec, 47)
    out = ctx.decode_attention(cache.K, cache.V, cache.lens, q, block_table=cache.block_table)
    assert ctx.get_error()[0] == tri.TRI_OK
    check_attention(cache, q, out, label=f"{name} after prune")
    ctx.close()


def test_attention_refused_sequence_is_not_written():
    spec = ts.CacheSpec(name="att_bad", head_dim=128, group=4, n_kv_heads=2, n_layers=1, batch=3,
                        rope_base=1e6, budget=64, offsets=(1,), positions="from_zero",
                        lens=(100, 100, 100), key_sigma=(0.1, 0.6), cap=128)
    cache = ts.make_cache(spec, 48).to("cuda")
    q = _queries(spec, 49)
    cache.lens[1] = 129  # above the capacity
    ctx = gu.context_for(cache)
    out = torch.full(q.shape, float("nan"), device="cuda")
    ctx.decode_attention(cache.K, cache.V, cache.lens, q, out=out)
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == tri.TRI_DEV_LEN_GT_CAP and cache.unit_index(unit)[1] == 1
    assert torch.isnan(out[:, 1]).all()
    lens = cache.lens_host.copy()
    lens[1] = 0
    o = out.clone()
    o[:, 1] = 0.0
    check_attention(cache, q, o, lens=lens, label="others")
    ctx.close()


@pytest.mark.parametrize("page_size", [32, 48])
def test_attention_paged_odd_pages(page_size):
    """Pages of 32 and 48 slots (GQA 8): a 16-row stage never crosses a page."""
    spec = ts.replace(ts.WORKLOADS["qwen3_32b_paged_ragged"], n_layers=1, batch=3, lens=(400, 257, 48),
                      page_size=page_size, budget=100, cap=480)
    cache = ts.make_cache(spec, 50).to("cuda")
    q = _queries(spec, 51)
    ctx = gu.context_for(cache)
    out = ctx.decode_attention(cache.K, cache.V, cache.lens, q, block_table=cache.block_table)
    assert ctx.get_error()[0] == tri.TRI_OK
    check_attention(cache, q, out, label=f"paged{page_size}")
    ctx.close()


def test_attention_layer_range():
    """A call on a sub-range of the layers (layer_begin) attends over exactly those layers (its
    units may be split into chunks differently from a full call, so each result is checked
    against the oracle, not against the other bit for bit)."""
    spec = ts.CacheSpec(name="att_layers", head_dim=128, group=4, n_kv_heads=2, n_layers=3, batch=2,
                        rope_base=1e6, budget=64, offsets=(1,), positions="from_zero",
                        lens=(300, 77), key_sigma=(0.1, 0.6), cap=320)
    cache = ts.make_cache(spec, 52).to("cuda")
    q = _queries(spec, 53)
    ctx = gu.context_for(cache)
    full = ctx.decode_attention(cache.K, cache.V, cache.lens, q)
    part = ctx.decode_attention(cache.K[1:3].contiguous(), cache.V[1:3].contiguous(), cache.lens,
                                q[1:3].contiguous(), layer_begin=1)
    assert ctx.get_error()[0] == tri.TRI_OK
    check_attention(cache, q, full, label="all layers")
    sub = ts.Cache(ts.replace(spec, n_layers=2), cache.K[1:3], cache.V[1:3], cache.pos[1:3], cache.lens,
                   cache.t, None, 0, cache.cap, (cache.q_mean[1:3], cache.q_norm_mean[1:3], cache.R[1:3],
                                                 cache.offsets))
    check_attention(sub, q[1:3], part, label="layers 1-2")
    ctx.close()
