"""Calibration statistics on disk.

The statistics are the only state of TriAttention that outlives a process: they come from an
offline calibration pass over a small batch of tokens and are loaded once per model (the
deep-dive page on TriAttention: §3.4 describes the one-off calibration, and the calibrator of
its §4.1 saves and reloads the statistics with torch's serializer). The C library does no file
I/O, so this module keeps them in a plain file and hands them to ``tri_calibrate_load``:

* ``.npz`` (numpy) or ``.pt`` (a dict of CPU tensors, read with ``weights_only=True``);
* arrays: ``q_mean`` fp32 [L][Hq][d] (the pre-RoPE query centre, the keys' dim layout),
  ``q_norm_mean`` fp32 [L][Hq][d/2] (E|q_f|), ``R`` fp32 [L][Hq][d/2] (|E q_f| / E|q_f|),
  ``offsets`` int64 [n] (future offsets delta);
* scalars: ``format`` (1), ``n_kv_heads``, ``group``, ``rope_base``, ``layout`` (0 half,
  1 interleaved).

``load`` checks shapes, types, ranges and finiteness before anything reaches a context, with the
same rules as ``tri_calibrate_load`` (head_dim 64 or 128, group 1/2/4/8, rope_base > 0). Nothing
here computes on the scoring path.
"""
from __future__ import annotations

import dataclasses
import os

import numpy as np

FORMAT = 1


class StatsError(ValueError):
    pass


@dataclasses.dataclass
class CalibStats:
    q_mean: np.ndarray        # fp32 [L][Hq][d]
    q_norm_mean: np.ndarray   # fp32 [L][Hq][d/2]
    R: np.ndarray             # fp32 [L][Hq][d/2]
    offsets: np.ndarray       # int64 [n]
    n_kv_heads: int
    group: int
    rope_base: float
    layout: int = 0

    @property
    def n_layers(self) -> int:
        return int(self.q_mean.shape[0])

    @property
    def head_dim(self) -> int:
        return int(self.q_mean.shape[2])

    def validate(self) -> "CalibStats":
        qm, qn, R, off = self.q_mean, self.q_norm_mean, self.R, self.offsets
        for name, a, dt in (("q_mean", qm, np.float32), ("q_norm_mean", qn, np.float32), ("R", R, np.float32),
                            ("offsets", off, np.int64)):
            if not isinstance(a, np.ndarray) or a.dtype != dt:
                raise StatsError(f"{name}: expected a numpy {np.dtype(dt).name} array")
        if qm.ndim != 3:
            raise StatsError("q_mean: expected [n_layers][n_q_heads][head_dim]")
        L, Hq, d = qm.shape
        if d not in (64, 128):
            raise StatsError(f"head_dim {d} not in (64, 128)")
        if self.group not in (1, 2, 4, 8):
            raise StatsError(f"group {self.group} not in (1, 2, 4, 8)")
        if self.n_kv_heads < 1 or Hq != self.n_kv_heads * self.group:
            raise StatsError(f"{Hq} query heads != n_kv_heads {self.n_kv_heads} x group {self.group}")
        if L < 1:
            raise StatsError("no layers")
        for name, a in (("q_norm_mean", qn), ("R", R)):
            if a.shape != (L, Hq, d // 2):
                raise StatsError(f"{name}: shape {a.shape} != {(L, Hq, d // 2)}")
        if off.ndim != 1 or off.size < 1:
            raise StatsError("offsets: expected a non-empty 1-D array")
        if not (np.isfinite(qm).all() and np.isfinite(qn).all() and np.isfinite(R).all()):
            raise StatsError("non-finite statistics")
        if (qn < 0).any() or (R < 0).any() or (R > 1.0 + 1e-6).any():
            raise StatsError("E|q_f| must be >= 0 and R_f in [0, 1]")
        if not (self.rope_base > 0.0 and np.isfinite(self.rope_base)):
            raise StatsError(f"rope_base {self.rope_base} must be positive and finite")
        if self.layout not in (0, 1):
            raise StatsError(f"layout {self.layout} not in (0, 1)")
        return self

    def load_into(self, ctx) -> None:
        """tri_calibrate_load on a TriContext."""
        self.validate()
        ctx.calibrate_load(self.n_layers, self.n_kv_heads, self.group, self.head_dim, self.rope_base,
                           self.layout, self.q_mean, self.q_norm_mean, self.R, self.offsets)


def _fields(s: CalibStats) -> dict:
    return dict(format=np.int64(FORMAT), q_mean=s.q_mean, q_norm_mean=s.q_norm_mean, R=s.R,
                offsets=s.offsets, n_kv_heads=np.int64(s.n_kv_heads), group=np.int64(s.group),
                rope_base=np.float64(s.rope_base), layout=np.int64(s.layout))


def save(path: str, stats: CalibStats) -> None:
    """Write the statistics (validated first) to ``path`` (.npz or .pt)."""
    stats.validate()
    f = _fields(stats)
    tmp = path + ".tmp"
    if path.endswith(".pt"):
        import torch
        torch.save({k: torch.from_numpy(np.asarray(v)) for k, v in f.items()}, tmp)
    else:
        with open(tmp, "wb") as fh:  # a file object keeps numpy from appending ".npz"
            np.savez(fh, **f)
    os.replace(tmp, path)  # a reader never sees a half-written file


def load(path: str) -> CalibStats:
    """Read and validate statistics written by ``save``."""
    if path.endswith(".pt"):
        import torch
        raw = torch.load(path, map_location="cpu", weights_only=True)
        f = {k: v.numpy() for k, v in raw.items()}
    else:
        with np.load(path, allow_pickle=False) as z:
            f = {k: z[k] for k in z.files}
    need = ("format", "q_mean", "q_norm_mean", "R", "offsets", "n_kv_heads", "group", "rope_base", "layout")
    missing = [k for k in need if k not in f]
    if missing:
        raise StatsError(f"missing fields: {missing}")
    if int(f["format"]) != FORMAT:
        raise StatsError(f"format {int(f['format'])} != {FORMAT}")
    s = CalibStats(q_mean=np.ascontiguousarray(f["q_mean"]), q_norm_mean=np.ascontiguousarray(f["q_norm_mean"]),
                   R=np.ascontiguousarray(f["R"]), offsets=np.ascontiguousarray(f["offsets"]),
                   n_kv_heads=int(f["n_kv_heads"]), group=int(f["group"]), rope_base=float(f["rope_base"]),
                   layout=int(f["layout"]))
    return s.validate()


def from_estimate(q_mean, q_norm_mean, R, offsets, n_kv_heads: int, group: int, rope_base: float,
                  layout: int = 0) -> CalibStats:
    """Statistics from ``tri_calibrate_estimate``'s outputs (CUDA or CPU tensors, or arrays)."""
    def host(a, dt):
        if hasattr(a, "detach"):
            a = a.detach().to("cpu").numpy()
        return np.ascontiguousarray(np.asarray(a, dtype=dt))
    return CalibStats(q_mean=host(q_mean, np.float32), q_norm_mean=host(q_norm_mean, np.float32),
                      R=host(R, np.float32), offsets=host(offsets, np.int64), n_kv_heads=int(n_kv_heads),
                      group=int(group), rope_base=float(rope_base), layout=int(layout)).validate()
