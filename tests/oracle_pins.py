"""Checks that pin the fp64 oracle to things other than itself.

Each ``pin_*`` function takes a loaded oracle library handle and raises
AssertionError when the oracle disagrees with what the TriAttention pages and
the mathematics fix:

* worked examples small enough to check by hand (``golden/hand_examples.json``);
* the closed form the method rests on: with every query at its centre (R = 1,
  so the norm term vanishes) the trigonometric score equals the mean over the
  future offsets of the real dot product of the RoPE-rotated query centre and
  the stored key, computed here from the textbook 2x2 rotation per band;
* invariants: the score does not depend on the key positions once the stored
  keys and t are fixed (positions cancel between un-rotation and distance);
  moving t by c equals rotating the query centres by c; the norm term does
  not change when a key band is rotated; z has mean 0 and variance 1 per
  head; scaling every query statistic by c > 0 leaves z and the kept set alone;
* brute force on tiny inputs: the kept set is the lexicographically smallest
  of the B-subsets with the largest sum of max-z.

The calibration statistics (E[q_f], E|q_f| and R_f per band from query samples) are
pinned by a hand example (``golden/calibration_example.json``) and closed forms:
identical tokens give R = 1, opposite tokens R = 0, two tokens of equal modulus at an
angle theta give R = cos(theta / 2); repeating the token set changes nothing, scaling it
by 2 scales the centre and the mean modulus and leaves R alone, and the two rotary
layouts agree once the dims are permuted.

The mutation test plants plausible mistakes in copies of the oracle and checks
that each one trips at least one of these pins.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
LAYOUTS = {"half": oracle.HALF, "interleaved": oracle.INTERLEAVED}


def _bf16_bits(x):
    """Round fp64 values to bf16 (round to nearest even) and return the bits."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _bf16_value(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def _band_pairs(d, layout):
    F = d // 2
    if layout == oracle.HALF:
        return [(f, f + F) for f in range(F)]
    return [(2 * f, 2 * f + 1) for f in range(F)]


def rope_rotate(x, m, base, layout):
    """Textbook RoPE: rotate each band (a, b) of the real vector x by m * base^(-2f/d)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    out = x.copy()
    for f, (a, b) in enumerate(_band_pairs(d, layout)):
        th = m * base ** (-2.0 * f / d)
        rot = np.array([[math.cos(th), -math.sin(th)], [math.sin(th), math.cos(th)]])
        out[..., a], out[..., b] = (rot[0, 0] * x[..., a] + rot[0, 1] * x[..., b],
                                    rot[1, 0] * x[..., a] + rot[1, 1] * x[..., b])
    return out


def _rand_unit(rng, d, G, N, layout, base, r_one=False):
    F = d // 2
    # the statistics enter as fp32 (as at the library boundary): draw them fp32-exact
    q_mean = rng.standard_normal((G, d)).astype(np.float32).astype(np.float64)
    pairs = _band_pairs(d, layout)
    mag = np.stack([np.hypot(q_mean[:, a], q_mean[:, b]) for a, b in pairs], axis=1)
    R = np.ones((G, F)) if r_one else rng.uniform(0.5, 1.0, (G, F))
    q_norm = (mag / R).astype(np.float32).astype(np.float64)
    R = R.astype(np.float32).astype(np.float64)
    K = _bf16_bits(rng.standard_normal((N, d)) + rng.standard_normal(d))
    pos = np.sort(rng.choice(4 * N + 64, N, replace=False)).astype(np.int32)
    t = int(pos[-1]) + 1 + int(rng.integers(0, 5))
    return q_mean, q_norm, R, K, pos, t


def _expr(e):
    return float(eval(e, {"__builtins__": {}}, {"math": math}))


def pin_hand_examples(L):
    with open(os.path.join(HERE, "golden", "hand_examples.json")) as fh:
        g = json.load(fh)
    for ex in g["scores"]:
        K = _bf16_bits(np.array(ex["K"], dtype=np.float64))
        assert np.array_equal(_bf16_value(K), np.array(ex["K"])), ex["name"]
        s, _, _ = oracle.unit_scores(K, ex["pos"], ex["t"], ex["q_mean"], ex["q_norm"], ex["R"],
                                     ex["offsets"], ex["base"], LAYOUTS[ex["layout"]], L=L)
        want = np.array([_expr(e) for e in ex["expect"]])
        assert np.allclose(s[:, 0], want, rtol=0, atol=1e-12), (ex["name"], s[:, 0], want)
    for ex in g["scores_max"]:
        K = _bf16_bits(np.array(ex["K"], dtype=np.float64))
        assert np.array_equal(_bf16_value(K), np.array(ex["K"])), ex["name"]
        s, _, _ = oracle.unit_scores(K, ex["pos"], ex["t"], ex["q_mean"], ex["q_norm"], ex["R"],
                                     ex["offsets"], ex["base"], LAYOUTS[ex["layout"]], L=L, combine="max")
        want = np.array([_expr(e) for e in ex["expect"]])
        assert np.allclose(s[:, 0], want, rtol=0, atol=1e-12), (ex["name"], s[:, 0], want)
    for ex in g["zmax"]:
        z, zm = oracle.zmax(np.array(ex["s"]), L=L)
        assert np.allclose(z[0], [_expr(e) for e in ex["expect_z0"]], atol=1e-12), ex["name"]
        assert np.allclose(zm, [_expr(e) for e in ex["expect_zmax"]], atol=1e-12), ex["name"]
        for B, kept in ex["keep"].items():
            got = oracle.select(zm, int(B), L=L)
            assert got.tolist() == kept, (ex["name"], B, got, kept)


def pin_rope_dot_closed_form(L, seed=0):
    """R = 1: score == mean_delta RoPE(qbar, t + delta) . k~ (stored key), to 1e-9 of scale."""
    rng = np.random.default_rng(seed)
    for d, base, offsets in ((8, 1e4, [0]), (64, 1e4, [1 << i for i in range(11)]),
                             (128, 1e6, [1 << i for i in range(17)])):
        for layout in (oracle.HALF, oracle.INTERLEAVED):
            G, N = 3, 17
            q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, layout, base, r_one=True)
            s, trig, norm = oracle.unit_scores(K, pos, t, q_mean, q_norm, R, offsets, base, layout, L=L)
            kval = _bf16_value(K)
            want = np.zeros((G, N))
            for h in range(G):
                for dl in offsets:
                    qrot = rope_rotate(q_mean[h], t + dl, base, layout)
                    want[h] += kval @ qrot
                want[h] /= len(offsets)
            scale = np.abs(want).max()
            assert np.abs(norm).max() == 0.0
            assert np.abs(s - want).max() <= 1e-9 * scale, (d, layout, np.abs(s - want).max(), scale)


def pin_positions_cancel(L, seed=1):
    """Fixed stored keys and t: moving the key positions must not change any score."""
    rng = np.random.default_rng(seed)
    for layout in (oracle.HALF, oracle.INTERLEAVED):
        d, G, N, base = 128, 4, 23, 1e6
        off = [1 << i for i in range(17)]
        q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, layout, base)
        s1, _, _ = oracle.unit_scores(K, pos, t, q_mean, q_norm, R, off, base, layout, L=L)
        pos2 = np.sort(rng.choice(t, N, replace=False)).astype(np.int32)
        s2, _, _ = oracle.unit_scores(K, pos2, t, q_mean, q_norm, R, off, base, layout, L=L)
        assert np.abs(s1 - s2).max() <= 1e-9 * np.abs(s1).max(), np.abs(s1 - s2).max()


def pin_t_shift_is_query_rotation(L, seed=2):
    """Score at t + c with centres qbar equals score at t with centres RoPE(qbar, c)."""
    rng = np.random.default_rng(seed)
    for layout in (oracle.HALF, oracle.INTERLEAVED):
        d, G, N, base, c = 64, 2, 19, 1e4, 37
        off = [1 << i for i in range(11)]
        q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, layout, base)
        s1, tr1, _ = oracle.unit_scores(K, pos, t + c, q_mean, q_norm, R, off, base, layout, L=L)
        q_rot = np.stack([rope_rotate(q_mean[h], c, base, layout) for h in range(G)])
        s2, tr2, _ = oracle.unit_scores(K, pos, t, q_rot, q_norm, R, off, base, layout, L=L)
        # the rotated centres pass through fp32 at the interface: 1e-6 of scale
        assert np.abs(tr1 - tr2).max() <= 1e-6 * np.abs(tr1).max()
        assert np.abs(s1 - s2).max() <= 1e-6 * np.abs(s1).max()


def pin_norm_rotation_invariant_and_linear(L, seed=3):
    """The norm term ignores band rotations of the key and is linear in the weights."""
    rng = np.random.default_rng(seed)
    for layout in (oracle.HALF, oracle.INTERLEAVED):
        d, G, N, base = 16, 2, 9, 1e4
        q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, layout, base)
        zero = np.zeros_like(q_mean)
        _, tr, n1 = oracle.unit_scores(K, pos, t, zero, q_norm, R, [1, 2], base, layout, L=L)
        assert np.abs(tr).max() == 0.0
        # rotate every band of every key by a quarter turn: (a, b) -> (-b, a) is exact in bf16
        K2 = K.copy()
        for a, b in _band_pairs(d, layout):
            K2[:, a] = K[:, b] ^ np.uint16(0x8000)
            K2[:, b] = K[:, a]
        _, _, n2 = oracle.unit_scores(K2, pos, t, zero, q_norm, R, [1, 2], base, layout, L=L)
        assert np.abs(n1 - n2).max() <= 1e-12 * np.abs(n1).max()
        # linearity in the weight (1 - R) E|q|
        _, _, na = oracle.unit_scores(K, pos, t, zero, q_norm, np.zeros_like(R), [1], base, layout, L=L)
        _, _, nb = oracle.unit_scores(K, pos, t, zero, q_norm, 0.75 * np.ones_like(R), [1], base, layout, L=L)
        assert np.abs(nb - 0.25 * na).max() <= 1e-12 * np.abs(na).max()
        # R = 1 removes it
        _, _, nc = oracle.unit_scores(K, pos, t, zero, q_norm, np.ones_like(R), [1], base, layout, L=L)
        assert np.abs(nc).max() == 0.0


def pin_z_invariants(L, seed=4):
    rng = np.random.default_rng(seed)
    for G, N in ((1, 5), (4, 300), (8, 77)):
        s = rng.standard_normal((G, N)) * rng.uniform(0.1, 50, (G, 1)) + rng.uniform(-9, 9, (G, 1))
        z, zm = oracle.zmax(s, L=L)
        assert np.abs(z.mean(axis=1)).max() <= 1e-12
        assert np.abs((z * z).mean(axis=1) - 1.0).max() <= 1e-12
        assert np.array_equal(zm, z.max(axis=0))
        # flat head gives zero z
        s2 = s.copy(); s2[0] = 3.25
        z2, _ = oracle.zmax(s2, L=L)
        assert np.all(z2[0] == 0.0)


def pin_scale_invariance(L, seed=5):
    """Scaling qbar and E|q| by c > 0 scales every score by c: z and the kept set do not move."""
    rng = np.random.default_rng(seed)
    d, G, N, base, B = 64, 4, 200, 1e4, 37
    off = [1 << i for i in range(11)]
    q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, oracle.HALF, base)
    # keep 2.5 * stats exact in fp32: round the stats to 2^-10 steps first
    q_mean = np.round(q_mean * 1024) / 1024
    q_norm = np.round(q_norm * 1024) / 1024
    V = K[::-1].copy()
    a = oracle.prune_unit(K, V, pos, t, q_mean, q_norm, R, off, base, B, L=L)
    b = oracle.prune_unit(K, V, pos, t, 2.5 * q_mean, 2.5 * q_norm, R, off, base, B, L=L)
    assert np.abs(b["s"] - 2.5 * a["s"]).max() <= 1e-12 * np.abs(b["s"]).max()
    assert np.abs(a["z"] - b["z"]).max() <= 1e-9
    assert np.array_equal(a["kept"], b["kept"])


def pin_select_brute_force(L, seed=6):
    """Kept set == lexicographically smallest B-subset with the largest sum (integer zmax, many ties)."""
    rng = np.random.default_rng(seed)
    for trial in range(60):
        N = int(rng.integers(1, 11))
        B = int(rng.integers(1, 12))
        zm = rng.integers(-3, 4, N).astype(np.float64)
        got = oracle.select(zm, B, L=L).tolist()
        M = min(N, B)
        best = None
        for sub in itertools.combinations(range(N), M):
            key = (-sum(zm[list(sub)]), sub)
            if best is None or key < best:
                best = key
        assert got == list(best[1]), (zm, B, got, best)


def pin_compaction(L, seed=7):
    rng = np.random.default_rng(seed)
    d, G, N, base = 32, 2, 150, 1e4
    q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, oracle.HALF, base)
    V = _bf16_bits(rng.standard_normal((N, d)))
    for B in (1, 40, 149, 150, 400):
        r = oracle.prune_unit(K, V, pos, t, q_mean, q_norm, R, [1, 4], base, B, L=L)
        kept = r["kept"]
        assert len(kept) == min(N, B)
        assert np.all(np.diff(kept) > 0)
        assert np.array_equal(r["K"], K[kept]) and np.array_equal(r["V"], V[kept])
        assert np.array_equal(r["pos"], pos[kept])
        # kept keys dominate dropped keys (ties to the lower slot)
        drop = np.setdiff1d(np.arange(N), kept)
        if len(drop) and len(kept):
            assert r["zmax"][kept].min() >= r["zmax"][drop].max()


def pin_max_over_delta(L, seed=9):
    """The variant that combines the offsets by the maximum: with R = 1 it equals max over delta
    of the textbook-RoPE dot product; with one offset it equals the mean mode; it is never below
    the mean mode; the norm term is the same in both modes; positions still cancel."""
    rng = np.random.default_rng(seed)
    for d, base, offsets in ((8, 1e4, [1, 2]), (64, 1e4, [1 << i for i in range(11)]),
                             (128, 1e6, [1 << i for i in range(17)])):
        for layout in (oracle.HALF, oracle.INTERLEAVED):
            G, N = 3, 17
            q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, layout, base, r_one=True)
            s, trig, norm = oracle.unit_scores(K, pos, t, q_mean, q_norm, R, offsets, base, layout, L=L,
                                               combine="max")
            kval = _bf16_value(K)
            want = np.full((G, N), -np.inf)
            for h in range(G):
                for dl in offsets:
                    want[h] = np.maximum(want[h], kval @ rope_rotate(q_mean[h], t + dl, base, layout))
            scale = np.abs(want).max()
            assert np.abs(norm).max() == 0.0
            assert np.abs(s - want).max() <= 1e-9 * scale, (d, layout, np.abs(s - want).max(), scale)
            # R < 1: max >= mean, identical norm terms, one offset gives the mean mode exactly
            q_mean, q_norm, R, K, pos, t = _rand_unit(rng, d, G, N, layout, base)
            s_mx, tr_mx, nm_mx = oracle.unit_scores(K, pos, t, q_mean, q_norm, R, offsets, base, layout, L=L,
                                                    combine="max")
            s_mn, tr_mn, nm_mn = oracle.unit_scores(K, pos, t, q_mean, q_norm, R, offsets, base, layout, L=L)
            assert np.all(tr_mx >= tr_mn - 1e-12 * np.abs(tr_mn).max())
            assert np.array_equal(nm_mx, nm_mn)
            one = oracle.unit_scores(K, pos, t, q_mean, q_norm, R, offsets[-1:], base, layout, L=L, combine="max")
            one_mean = oracle.unit_scores(K, pos, t, q_mean, q_norm, R, offsets[-1:], base, layout, L=L)
            assert np.array_equal(one[0], one_mean[0])
            # positions cancel: the same stored keys at other positions, same t
            pos2 = np.sort(rng.choice(int(pos[-1]) + 1, N, replace=False)).astype(np.int32)
            s2 = oracle.unit_scores(K, pos2, t, q_mean, q_norm, R, offsets, base, layout, L=L, combine="max")[0]
            assert np.abs(s2 - s_mx).max() <= 1e-9 * np.abs(s_mx).max()


def pin_prune_batch_matches_units(L, seed=12):
    """The batch driver (threads over units, one flat buffer per argument) gives, unit by
    unit, what the single-unit pass gives on that unit's own slice: same kept slots, count and
    max-z, for ragged lengths (0, 1, B, B + 1 and random), groups 1/4/8, both head sizes and
    rotary layouts, and both ways of combining the offsets. A wrong per-unit offset into any
    of the flat inputs or outputs reads or writes another unit's data and fails here."""
    rng = np.random.default_rng(seed)
    cases = ((64, 1, oracle.HALF, "mean"), (64, 4, oracle.INTERLEAVED, "max"),
             (128, 8, oracle.HALF, "max"), (128, 4, oracle.INTERLEAVED, "mean"),
             (128, 2, oracle.HALF, "mean"))
    for d, G, layout, combine in cases:
        base = 1e4 if d == 64 else 1e6
        offsets = [1 << i for i in range(11 if d == 64 else 17)]
        B, S = 13, 40
        lens = [0, 1, B, B + 1, S] + [int(x) for x in rng.integers(2, S + 1, 2)]
        U = len(lens)
        units = [_rand_unit(rng, d, G, S, layout, base) for _ in range(U)]
        Kb = np.stack([u[3] for u in units])
        Pb = np.stack([u[4] for u in units])
        qm = np.stack([u[0] for u in units])
        qn = np.stack([u[1] for u in units])
        RR = np.stack([u[2] for u in units])
        # t differs per unit: each unit's own t (its positions all lie below it)
        tt = np.array([u[5] + 7 * i for i, u in enumerate(units)], np.int64)
        kept, nk, zm, sc = oracle.prune_batch(Kb, Pb, np.array(lens, np.int32), tt, qm, qn, RR, offsets, base, B,
                                              layout, n_threads=2, want_zmax=True, L=L, combine=combine,
                                              want_scores=True)
        for u, n in enumerate(lens):
            assert nk[u] == min(n, B), (d, G, combine, u, nk[u], n)
            if n == 0:
                continue
            V = Kb[u, :n][::-1].copy()
            one = oracle.prune_unit(Kb[u, :n], V, Pb[u, :n], int(tt[u]), qm[u], qn[u], RR[u], offsets, base, B,
                                    layout, L=L, combine=combine)
            assert np.array_equal(kept[u, :nk[u]], one["kept"]), (d, G, combine, u)
            assert np.array_equal(zm[u, :n], one["zmax"]), (d, G, combine, u)
            assert np.array_equal(sc[u, :, :n], one["s"]), (d, G, combine, u)


def pin_select_f32(L, seed=13):
    """Selection on fp32 max-z values: the B largest, ties to the lower slot, returned in
    ascending slot order, checked against numpy's lexicographic sort on (-z, slot) and against
    the fp64 selection of the same (exactly widened) values. Inputs carry many exact ties and
    neighbours one fp32 ulp apart."""
    rng = np.random.default_rng(seed)
    for trial in range(40):
        N = int(rng.integers(1, 300))
        B = int(rng.integers(1, N + 20))
        z = rng.integers(-6, 7, N).astype(np.float32) * np.float32(0.375)
        bump = rng.random(N) < 0.3
        z[bump] = np.nextafter(z[bump], np.float32(np.inf))
        got = oracle.select(z, B, L=L)
        assert got.dtype == np.int32
        order = np.lexsort((np.arange(N), -z.astype(np.float64)))
        want = np.sort(order[:min(N, B)])
        assert np.array_equal(got, want), (N, B)
        assert np.array_equal(got, oracle.select(z.astype(np.float64), B, L=L))


def _calib_tokens(bands, d, layout):
    """[T][d] real vectors from [T][F][2] band samples, in the given rotary layout."""
    bands = np.asarray(bands, dtype=np.float64)
    T, F, _ = bands.shape
    x = np.zeros((T, d))
    for f, (re, im) in enumerate(_band_pairs(d, layout)):
        x[:, re] = bands[:, f, 0]
        x[:, im] = bands[:, f, 1]
    return x


def _calibrate(L, x, layout):
    """Oracle statistics of samples x [T][d] (one layer, one head), fp64 band views."""
    T, d = x.shape
    qm, qn, R = oracle.calibrate(_bf16_bits(x).reshape(1, T, 1, d), layout, L=L)
    pairs = _band_pairs(d, layout)
    cm = np.array([[qm[0, 0, re], qm[0, 0, im]] for re, im in pairs])
    return cm, qn[0, 0], R[0, 0]


def pin_calibrate_hand_example(L):
    with open(os.path.join(HERE, "golden", "calibration_example.json")) as fh:
        g = json.load(fh)
    for name, layout in LAYOUTS.items():
        cm, qn, R = _calibrate(L, _calib_tokens(g["bands"], 4, layout), layout)
        want_cm = np.array([[_expr(v) for v in b] for b in g["q_mean_bands"]])
        assert np.allclose(cm, want_cm, rtol=0, atol=1e-15), (name, cm)
        assert np.allclose(qn, [_expr(v) for v in g["q_norm_mean"]], rtol=0, atol=1e-14), (name, qn)
        assert np.allclose(R, [_expr(v) for v in g["R"]], rtol=0, atol=1e-15), (name, R)


def pin_calibrate_closed_forms(L):
    """Identical tokens: R = 1 (0 for an all-zero band); opposite tokens: R = 0; two tokens of
    equal modulus at angle theta: R = cos(theta / 2) (Pythagorean samples, exact in bf16)."""
    # identical tokens, one band all zero
    one = [[3.0, 4.0], [0.0, 0.0], [-1.5, 2.0], [5.0, -12.0]]
    cm, qn, R = _calibrate(L, _calib_tokens([one] * 5, 8, oracle.HALF), oracle.HALF)
    assert np.allclose(cm, one, rtol=0, atol=1e-15)
    assert np.allclose(qn, [5.0, 0.0, 2.5, 13.0], rtol=0, atol=1e-14)
    assert np.allclose(R, [1.0, 0.0, 1.0, 1.0], rtol=0, atol=1e-15), R
    # opposite tokens
    opp = [[[3.0, 4.0], [8.0, -15.0]], [[-3.0, -4.0], [-8.0, 15.0]]]
    cm, qn, R = _calibrate(L, _calib_tokens(opp, 4, oracle.INTERLEAVED), oracle.INTERLEAVED)
    assert np.allclose(cm, 0.0, atol=1e-15) and np.allclose(R, 0.0, atol=1e-15)
    assert np.allclose(qn, [5.0, 17.0], rtol=0, atol=1e-14)
    # two tokens of equal modulus: (a, b) and (b, a) for each Pythagorean pair, and (a, b), (a, -b)
    pairs = [(3.0, 4.0), (5.0, 12.0), (8.0, 15.0), (7.0, 24.0)]
    toks = [[[a, b] for a, b in pairs], [[b, a] for a, b in pairs]]
    cm, qn, R = _calibrate(L, _calib_tokens(toks, 8, oracle.HALF), oracle.HALF)
    for f, (a, b) in enumerate(pairs):
        r = math.hypot(a, b)
        cos_t = 2 * a * b / (r * r)
        assert abs(R[f] - math.sqrt((1 + cos_t) / 2)) < 1e-15, (f, R[f])
        assert abs(qn[f] - r) < 1e-13
    toks = [[[a, b] for a, b in pairs], [[a, -b] for a, b in pairs]]
    cm, qn, R = _calibrate(L, _calib_tokens(toks, 8, oracle.HALF), oracle.HALF)
    for f, (a, b) in enumerate(pairs):
        assert abs(R[f] - a / math.hypot(a, b)) < 1e-15, (f, R[f])


def pin_calibrate_invariants(L, seed=8):
    """Repeating the token set changes nothing; doubling every sample doubles E[q] and E|q|
    and keeps R; the two rotary layouts give the same statistics per band."""
    rng = np.random.default_rng(seed)
    T, F = 37, 16
    bands = _bf16_value(_bf16_bits(rng.normal(0.3, 1.0, (T, F, 2))))
    for layout in LAYOUTS.values():
        cm, qn, R = _calibrate(L, _calib_tokens(bands, 2 * F, layout), layout)
        cm2, qn2, R2 = _calibrate(L, _calib_tokens(np.concatenate([bands, bands, bands]), 2 * F, layout), layout)
        assert np.allclose(cm2, cm, rtol=1e-14, atol=1e-15) and np.allclose(qn2, qn, rtol=1e-14)
        assert np.allclose(R2, R, rtol=1e-13)
        cm3, qn3, R3 = _calibrate(L, _calib_tokens(2.0 * bands, 2 * F, layout), layout)
        assert np.allclose(cm3, 2 * cm, rtol=1e-14, atol=1e-15) and np.allclose(qn3, 2 * qn, rtol=1e-14)
        assert np.allclose(R3, R, rtol=1e-13)
        assert np.all((R >= 0) & (R <= 1 + 1e-15))
    ch, qh, Rh = _calibrate(L, _calib_tokens(bands, 2 * F, oracle.HALF), oracle.HALF)
    ci, qi, Ri = _calibrate(L, _calib_tokens(bands, 2 * F, oracle.INTERLEAVED), oracle.INTERLEAVED)
    assert np.array_equal(ch, ci) and np.array_equal(qh, qi) and np.array_equal(Rh, Ri)


def pin_attention_special_cases(L, seed=10):
    """Decode attention over kept rows: one key returns its value row exactly; identical keys
    weight every row equally (the mean of the values); permuting the kept rows (keys and
    values together) changes nothing; a zero query also gives the mean of the values."""
    r = np.random.default_rng(seed)
    d, G = 64, 2
    q = _bf16_bits(r.normal(size=(G, d)))
    K = _bf16_bits(r.normal(size=(9, d)))
    V = _bf16_bits(r.normal(size=(9, d)))
    one = oracle.decode_attention(q, K[:1], V[:1], L=L)
    assert np.array_equal(one, np.broadcast_to(_bf16_value(V[:1]), (G, d)))
    same = oracle.decode_attention(q, np.repeat(K[:1], 9, axis=0), V, L=L)
    assert np.abs(same - _bf16_value(V).mean(axis=0)).max() <= 1e-14
    zero = oracle.decode_attention(np.zeros_like(q), K, V, L=L)
    assert np.abs(zero - _bf16_value(V).mean(axis=0)).max() <= 1e-14
    perm = r.permutation(9)
    a = oracle.decode_attention(q, K, V, L=L)
    b = oracle.decode_attention(q, K[perm], V[perm], L=L)
    assert np.abs(a - b).max() <= 1e-14


def pin_attention_library(L, seed=11):
    """Against torch's scaled_dot_product_attention in float64 (an independent implementation
    of the same definition), for both head sizes and GQA groups of 1 and 4."""
    import torch
    r = np.random.default_rng(seed)
    for d, G, M in ((64, 1, 5), (128, 4, 300)):
        q = _bf16_bits(r.normal(scale=2.0, size=(G, d)))
        K = _bf16_bits(r.normal(size=(M, d)))
        V = _bf16_bits(r.normal(size=(M, d)))
        got = oracle.decode_attention(q, K, V, L=L)
        tq = torch.from_numpy(_bf16_value(q))[None, :, None, :]
        tk = torch.from_numpy(_bf16_value(K))[None, None].expand(1, G, M, d)
        tv = torch.from_numpy(_bf16_value(V))[None, None].expand(1, G, M, d)
        want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, :, 0, :].numpy()
        assert np.abs(got - want).max() <= 1e-12 * max(1.0, np.abs(want).max()), (d, G, M)


ALL_PINS = [pin_hand_examples, pin_rope_dot_closed_form, pin_positions_cancel,
            pin_t_shift_is_query_rotation, pin_norm_rotation_invariant_and_linear,
            pin_z_invariants, pin_scale_invariance, pin_select_brute_force, pin_compaction,
            pin_calibrate_hand_example, pin_calibrate_closed_forms, pin_calibrate_invariants,
            pin_max_over_delta, pin_attention_special_cases, pin_attention_library,
            pin_prune_batch_matches_units, pin_select_f32]
