"""ctypes wrapper around the fp64 CPU oracle (``oracle/tri_oracle.c``).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The product path (the
``rope_aware_key_tri_b200`` package and its CUDA library) never does, and the
two share no code.

Every function here is marshalling only; the arithmetic lives in the C file,
whose header cites the TriAttention passages each step follows.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

HALF = 0
INTERLEAVED = 1

_lib = None


def lib(path: str | None = None):
    """Load (building first if stale) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _bind(L):
    P = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    L.tri_oracle_unit_scores.argtypes = [i32, i32, i32, f64, P, i32, i64, P, P, P, P, P, i32, P, P, P]
    L.tri_oracle_unit_scores.restype = i32
    L.tri_oracle_zmax.argtypes = [i32, i32, P, P, P]
    L.tri_oracle_zmax.restype = i32
    L.tri_oracle_select.argtypes = [i32, i32, P, P]
    L.tri_oracle_select.restype = i32
    L.tri_oracle_select_f32.argtypes = [i32, i32, P, P]
    L.tri_oracle_select_f32.restype = i32
    L.tri_oracle_compact.argtypes = [i32, i32, P, P, P, P, P, P, P]
    L.tri_oracle_compact.restype = i32
    L.tri_oracle_prune_batch.argtypes = [i32, i32, i32, i32, i32, i32, f64, P, i32, P,
                                         P, P, P, P, P, P, P, P, P, P, i32]
    L.tri_oracle_prune_batch.restype = i32
    L.tri_oracle_prune_batch_max.argtypes = L.tri_oracle_prune_batch.argtypes
    L.tri_oracle_prune_batch_max.restype = i32
    L.tri_oracle_unit_scores_max.argtypes = L.tri_oracle_unit_scores.argtypes
    L.tri_oracle_unit_scores_max.restype = i32
    L.tri_oracle_calibrate.argtypes = [P, i32, i32, i32, i32, i32, P, P, P]
    L.tri_oracle_calibrate.restype = i32
    L.tri_oracle_decode_attention.argtypes = [i32, i32, i32, P, P, P, P]
    L.tri_oracle_decode_attention.restype = i32
    return L


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def unit_scores(K_bits, pos, t, q_mean, q_norm, R, offsets, base, layout=HALF, L=None, combine="mean"):
    """Per-head scores of one unit: returns (s, trig, norm), each fp64 [G][N].

    K_bits: uint16 [N][d] bf16 bits of the stored keys; pos: int [N];
    q_mean: [G][d]; q_norm, R: [G][d/2]; offsets: the future-offset set;
    combine: "mean" (the pass) or "max" over the offsets (the variant).
    """
    L = L or lib()
    fn = {"mean": L.tri_oracle_unit_scores, "max": L.tri_oracle_unit_scores_max}[combine]
    K_bits = _c(K_bits, np.uint16)
    N, d = K_bits.shape
    q_mean = _c(q_mean, np.float32).reshape(-1, d)
    G = q_mean.shape[0]
    q_norm = _c(q_norm, np.float32).reshape(G, d // 2)
    R = _c(R, np.float32).reshape(G, d // 2)
    pos = _c(pos, np.int32)
    off = _c(offsets, np.int64)
    s = np.empty((G, N)); tr = np.empty((G, N)); nm = np.empty((G, N))
    rc = fn(d, G, layout, float(base), _p(off), len(off), int(t),
            _p(q_mean), _p(q_norm), _p(R), _p(K_bits), _p(pos), N,
            _p(s), _p(tr), _p(nm))
    if rc != 0:
        raise ValueError("tri_oracle_unit_scores rejected its arguments")
    return s, tr, nm


def zmax(s, L=None):
    """(z [G][N], zmax [N]) from per-head scores s [G][N]."""
    L = L or lib()
    s = _c(s, np.float64)
    G, N = s.shape
    z = np.empty((G, N)); zm = np.empty(N)
    if L.tri_oracle_zmax(G, N, _p(s), _p(z), _p(zm)) != 0:
        raise ValueError("tri_oracle_zmax rejected its arguments")
    return z, zm


def select(zm, B, L=None):
    """Kept slots (ascending) of the top-B by zm, ties to the lower slot."""
    L = L or lib()
    f32 = np.asarray(zm).dtype == np.float32
    zm = _c(zm, np.float32 if f32 else np.float64)
    N = zm.shape[0]
    out = np.empty(max(1, min(N, B)), dtype=np.int32)
    fn = L.tri_oracle_select_f32 if f32 else L.tri_oracle_select
    m = fn(N, int(B), _p(zm), _p(out))
    if m < 0:
        raise ValueError("tri_oracle_select rejected its arguments")
    return out[:m]


def compact(kept, K_bits, V_bits, pos, L=None):
    """Rows gathered at ``kept``: (K [M][d], V [M][d], pos [M])."""
    L = L or lib()
    kept = _c(kept, np.int32)
    K_bits = _c(K_bits, np.uint16); V_bits = _c(V_bits, np.uint16); pos = _c(pos, np.int32)
    M = kept.shape[0]
    d = K_bits.shape[1]
    Ko = np.empty((M, d), np.uint16); Vo = np.empty((M, d), np.uint16); po = np.empty(M, np.int32)
    if L.tri_oracle_compact(d, M, _p(kept), _p(K_bits), _p(V_bits), _p(pos), _p(Ko), _p(Vo), _p(po)) != 0:
        raise ValueError("tri_oracle_compact rejected its arguments")
    return Ko, Vo, po


def prune_unit(K_bits, V_bits, pos, t, q_mean, q_norm, R, offsets, base, B, layout=HALF, L=None,
               combine="mean"):
    """The whole pass on one unit. Returns a dict with s, z, zmax, kept and the compacted rows.
    combine: how the offsets combine in the trigonometric score ("mean" or "max")."""
    s, tr, nm = unit_scores(K_bits, pos, t, q_mean, q_norm, R, offsets, base, layout, L, combine=combine)
    z, zm = zmax(s, L)
    kept = select(zm, B, L)
    Ko, Vo, po = compact(kept, K_bits, V_bits, pos, L)
    return dict(s=s, trig=tr, norm=nm, z=z, zmax=zm, kept=kept, K=Ko, V=Vo, pos=po)


def prune_batch(K_bits, pos, lens, t, q_mean, q_norm, R, offsets, base, B, layout=HALF,
                n_threads=0, want_zmax=False, L=None, combine="mean", want_scores=False):
    """Selection for many units at once (threads over units); combine "mean" or "max".

    K_bits [U][S][d] uint16, pos [U][S], lens [U], t [U], q_mean [U][G][d],
    q_norm/R [U][G][d/2]. Returns (kept [U][B] int32, n_kept [U], zmax or None), and with
    want_scores also the per-head scores s [U][G][S] as a fourth element.
    """
    L = L or lib()
    K_bits = _c(K_bits, np.uint16)
    U, S, d = K_bits.shape
    q_mean = _c(q_mean, np.float32)
    G = q_mean.shape[1]
    q_norm = _c(q_norm, np.float32); R = _c(R, np.float32)
    pos = _c(pos, np.int32); lens = _c(lens, np.int32); t = _c(t, np.int64)
    off = _c(offsets, np.int64)
    kept = np.zeros((U, B), np.int32); nk = np.zeros(U, np.int32)
    zm = np.zeros((U, S)) if want_zmax else None
    sc = np.zeros((U, G, S)) if want_scores else None
    fn = {"mean": L.tri_oracle_prune_batch, "max": L.tri_oracle_prune_batch_max}[combine]
    rc = fn(U, S, int(B), d, G, layout, float(base), _p(off), len(off), _p(t),
            _p(q_mean), _p(q_norm), _p(R), _p(K_bits), _p(pos), _p(lens),
            _p(sc), _p(zm), _p(kept), _p(nk), int(n_threads))
    if rc != 0:
        raise ValueError("tri_oracle_prune_batch rejected its arguments")
    return (kept, nk, zm, sc) if want_scores else (kept, nk, zm)


def calibrate(Q_bits, layout=HALF, L=None):
    """Calibration statistics from pre-RoPE query samples.

    Q_bits: uint16 [L][T][Hq][d] bf16 bits. Returns fp64 (q_mean [L][Hq][d],
    q_norm_mean [L][Hq][d/2], R [L][Hq][d/2]).
    """
    Lb = L or lib()
    Q_bits = _c(Q_bits, np.uint16)
    nl, T, Hq, d = Q_bits.shape
    qm = np.zeros((nl, Hq, d), dtype=np.float64)
    qn = np.zeros((nl, Hq, d // 2), dtype=np.float64)
    R = np.zeros((nl, Hq, d // 2), dtype=np.float64)
    rc = Lb.tri_oracle_calibrate(_p(Q_bits), nl, T, Hq, d, int(layout), _p(qm), _p(qn), _p(R))
    if rc != 0:
        raise ValueError("tri_oracle_calibrate: bad arguments")
    return qm, qn, R


def decode_attention(q_bits, K_bits, V_bits, L=None):
    """Scaled dot-product attention of the G query heads over the M kept rows of one unit.

    q_bits uint16 [G][d], K_bits / V_bits uint16 [M][d] (bf16 bits, post-RoPE query and keys).
    Returns fp64 [G][d].
    """
    Lb = L or lib()
    q_bits = _c(q_bits, np.uint16); K_bits = _c(K_bits, np.uint16); V_bits = _c(V_bits, np.uint16)
    G, d = q_bits.shape
    M = K_bits.shape[0]
    if K_bits.shape != (M, d) or V_bits.shape != (M, d):
        raise ValueError("K and V must be [M][d] like the query's d")
    out = np.zeros((G, d), dtype=np.float64)
    if Lb.tri_oracle_decode_attention(d, G, M, _p(q_bits), _p(K_bits), _p(V_bits), _p(out)) != 0:
        raise ValueError("tri_oracle_decode_attention: bad arguments")
    return out
