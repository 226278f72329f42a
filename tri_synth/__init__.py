"""Seeded synthetic KV caches and calibration statistics.

This module only draws inputs. It holds none of the scoring, z-score,
selection or compaction arithmetic; both the CUDA path (through the
``rope_aware_key_tri_b200`` binding) and the fp64 oracle under ``oracle/``
consume what it produces. The one piece of position-encoding arithmetic here
is the RoPE rotation that turns the drawn pre-RoPE keys into the post-RoPE
keys an inference engine stores: that is how the cache is made, not part of
the pruning pass.

Recipe (TriAttention pages: the Qwen3-shaped caches that stand in for the
AIME/MATH500 runs, which need model weights and datasets). Per layer, in this
order of draws from one ``torch.Generator`` seeded with ``seed``:

1. key centre ``c[g, :] ~ N(0, 1)`` per KV head and dim;
2. key noise scale ``sigma[g]``: fixed (``key_sigma``) or ``U[lo, hi]``;
3. pre-RoPE keys ``k = c + sigma * N(0, 1)`` for every slot, then rotated
   by RoPE at the slot's position (angles in fp64) and rounded RNE to bf16;
4. values ``V ~ N(0, 1)`` rounded to bf16;
5. for the periodic-prune layout, the kept positions of the previous prune
   (a sorted random subset of ``[0, t - recent)`` plus the last ``recent``);
6. query statistics per query head: centre ``qbar ~ N(0, 1)`` per dim,
   ``R_f ~ U[r_lo, 1]`` per band, and ``E|q_f| = |qbar_f| / R_f``.

Slots at or beyond a sequence's length hold NaN keys/values and position -1,
so any kernel that reads past ``lens`` breaks the results loudly.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch

HALF = 0          # band f pairs dims (f, f + d/2) -- Qwen / NeoX rotary layout
INTERLEAVED = 1   # band f pairs dims (2f, 2f + 1) -- GPT-J rotary layout

BF16_NAN_BITS = 0x7FC0


@dataclasses.dataclass(frozen=True)
class CacheSpec:
    """Shape and distribution of one synthetic pruning workload."""

    name: str
    head_dim: int
    group: int                      # query heads per KV head (GQA group)
    n_kv_heads: int
    n_layers: int
    batch: int
    rope_base: float
    budget: int
    offsets: tuple                  # future offsets delta
    positions: str                  # "end_at_t" | "from_zero" | "periodic"
    lens: tuple                     # per-sequence cached tokens, or ("uniform", lo, hi)
    t: tuple = ()                   # per-sequence query position, or ("uniform", lo, hi); "from_zero" uses t = len
    key_sigma: tuple = (0.3, 0.3)   # U[lo, hi] per (layer, KV head)
    r_lo: float = 0.5
    layout: int = HALF
    page_size: int = 0              # 0 = dense cache
    recent: int = 128               # periodic layout: newest tokens always present
    cap: int = 0                    # dense slots per unit (0 = max length)

    @property
    def n_q_heads(self) -> int:
        return self.n_kv_heads * self.group

    @property
    def n_bands(self) -> int:
        return self.head_dim // 2


def pow2_offsets(top: int) -> tuple:
    return tuple(1 << i for i in range(top + 1))


# The five Qwen3-shaped workloads of the TriAttention pages (Qwen3-8B: 36 layers,
# 8 KV heads, GQA 4, head_dim 128, base 1e6; Qwen3-32B: 64 layers, 64 query heads),
# budgets 2048/3072 and the 128-token pruning cadence.
WORKLOADS = {
    "tiny_d64_n256": CacheSpec(
        name="tiny_d64_n256", head_dim=64, group=4, n_kv_heads=1, n_layers=1, batch=1,
        rope_base=1e4, budget=64, offsets=pow2_offsets(10), positions="from_zero",
        lens=(256,), key_sigma=(0.3, 0.3)),
    "qwen3_8b_decode_b16_2176": CacheSpec(
        name="qwen3_8b_decode_b16_2176", head_dim=128, group=4, n_kv_heads=8, n_layers=1,
        batch=16, rope_base=1e6, budget=2048, offsets=pow2_offsets(16), positions="end_at_t",
        lens=(2176,) * 16, t=("uniform", 4096, 32768), key_sigma=(0.1, 0.6)),
    "qwen3_8b_periodic_36l_3200": CacheSpec(
        name="qwen3_8b_periodic_36l_3200", head_dim=128, group=4, n_kv_heads=8, n_layers=36,
        batch=8, rope_base=1e6, budget=3072, offsets=pow2_offsets(16), positions="periodic",
        lens=(3200,) * 8, t=(24576,) * 8, key_sigma=(0.1, 0.6)),
    "qwen3_8b_oneshot_32k_to_3072": CacheSpec(
        name="qwen3_8b_oneshot_32k_to_3072", head_dim=128, group=4, n_kv_heads=8, n_layers=36,
        batch=4, rope_base=1e6, budget=3072, offsets=pow2_offsets(16), positions="from_zero",
        lens=(32768,) * 4, key_sigma=(0.1, 0.6)),
    "qwen3_32b_paged_ragged": CacheSpec(
        name="qwen3_32b_paged_ragged", head_dim=128, group=8, n_kv_heads=8, n_layers=64,
        batch=32, rope_base=1e6, budget=2048, offsets=pow2_offsets(16), positions="from_zero",
        lens=("uniform", 2176, 32768), key_sigma=(0.1, 0.6), page_size=64),
}


def rope_omega(head_dim: int, base: float) -> np.ndarray:
    """RoPE angular frequency per band, omega_f = base^(-2f/d), in fp64."""
    f = np.arange(head_dim // 2, dtype=np.float64)
    return base ** (-2.0 * f / head_dim)


def _uniform_int(gen: torch.Generator, lo: int, hi: int, n: int) -> list:
    return torch.randint(lo, hi + 1, (n,), generator=gen).tolist()


def resolve_lens_t(spec: CacheSpec, gen: torch.Generator):
    """Per-sequence cache length and query position t (last cached position is t - 1)."""
    if spec.lens and spec.lens[0] == "uniform":
        lens = _uniform_int(gen, spec.lens[1], spec.lens[2], spec.batch)
    else:
        lens = list(spec.lens)
    if spec.positions == "from_zero":
        t = list(lens)
    elif spec.t and spec.t[0] == "uniform":
        t = _uniform_int(gen, spec.t[1], spec.t[2], spec.batch)
    else:
        t = list(spec.t)
    return lens, t


def _rotate(k_pre: torch.Tensor, pos: torch.Tensor, omega: torch.Tensor, layout: int) -> torch.Tensor:
    """Apply RoPE at integer positions ``pos`` (broadcast over the last dim of k_pre)."""
    F = k_pre.shape[-1] // 2
    ang = pos.to(torch.float64).unsqueeze(-1) * omega            # [..., N, F] fp64
    c = torch.cos(ang).to(k_pre.dtype)
    s = torch.sin(ang).to(k_pre.dtype)
    if layout == HALF:
        re, im = k_pre[..., :F], k_pre[..., F:]
    else:
        re, im = k_pre[..., 0::2], k_pre[..., 1::2]
    re2 = re * c - im * s
    im2 = re * s + im * c
    if layout == HALF:
        return torch.cat([re2, im2], dim=-1)
    return torch.stack([re2, im2], dim=-1).flatten(-2)


def _positions_for_layer(spec, gen, lens, t, cap, device):
    """int32 [batch, Hkv, cap] positions (-1 beyond len)."""
    H = spec.n_kv_heads
    pos = torch.full((spec.batch, H, cap), -1, dtype=torch.int32)
    for s in range(spec.batch):
        n = lens[s]
        if spec.positions == "from_zero":
            pos[s, :, :n] = torch.arange(n, dtype=torch.int32)
        elif spec.positions == "end_at_t":
            pos[s, :, :n] = torch.arange(t[s] - n, t[s], dtype=torch.int32)
        elif spec.positions == "periodic":
            old = n - spec.recent
            pool = t[s] - spec.recent
            for g in range(H):
                pick = torch.randperm(pool, generator=gen)[:old].sort().values.to(torch.int32)
                pos[s, g, :old] = pick
                pos[s, g, old:n] = torch.arange(pool, t[s], dtype=torch.int32)
        else:
            raise ValueError(spec.positions)
    return pos.to(device)


def make_stats(spec: CacheSpec, seed: int):
    """Calibration statistics (fp32 numpy): q_mean [L][Hq][d], q_norm_mean [L][Hq][F], R [L][Hq][F]."""
    gen = torch.Generator().manual_seed(seed * 7919 + 17)
    L, Hq, d, F = spec.n_layers, spec.n_q_heads, spec.head_dim, spec.n_bands
    qm = torch.randn((L, Hq, d), generator=gen, dtype=torch.float64)
    R = spec.r_lo + (1.0 - spec.r_lo) * torch.rand((L, Hq, F), generator=gen, dtype=torch.float64)
    if spec.layout == HALF:
        re, im = qm[..., :F], qm[..., F:]
    else:
        re, im = qm[..., 0::2], qm[..., 1::2]
    mag = torch.sqrt(re * re + im * im)
    qn = mag / R
    return (qm.to(torch.float32).numpy(), qn.to(torch.float32).numpy(),
            R.to(torch.float32).numpy(), np.asarray(spec.offsets, dtype=np.int64))


class Cache:
    """A generated cache. Tensors live on ``device``; see ``make_cache``."""

    def __init__(self, spec, K, V, pos, lens, t, block_table, n_pages, cap, stats):
        self.spec = spec
        self.K, self.V, self.pos = K, V, pos
        self.lens, self.t = lens, t
        self.block_table = block_table
        self.n_pages = n_pages
        self.cap = cap
        self.q_mean, self.q_norm_mean, self.R, self.offsets = stats

    @property
    def paged(self) -> bool:
        return self.block_table is not None

    def to(self, device) -> "Cache":
        """Move every tensor of the cache to ``device`` (in place); returns self."""
        self.K, self.V, self.pos = self.K.to(device), self.V.to(device), self.pos.to(device)
        self.lens, self.t = self.lens.to(device), self.t.to(device)
        if self.block_table is not None:
            self.block_table = self.block_table.to(device)
        return self

    def clone(self) -> "Cache":
        c = Cache(self.spec, self.K.clone(), self.V.clone(), self.pos.clone(), self.lens.clone(),
                  self.t.clone(), None if self.block_table is None else self.block_table.clone(),
                  self.n_pages, self.cap, (self.q_mean, self.q_norm_mean, self.R, self.offsets))
        return c

    @property
    def n_units(self) -> int:
        s = self.spec
        return s.n_layers * s.batch * s.n_kv_heads

    def unit_index(self, u: int):
        s = self.spec
        g = u % s.n_kv_heads
        b = (u // s.n_kv_heads) % s.batch
        l = u // (s.n_kv_heads * s.batch)
        return l, b, g

    def unit_rows(self, u: int):
        """(K bits uint16 [n][d], V bits uint16 [n][d], pos int32 [n]) of one unit, logical order, on host."""
        s = self.spec
        l, b, g = self.unit_index(u)
        n = int(self.lens_host[b])
        if not self.paged:
            k = self.K[l, b, g, :n]
            v = self.V[l, b, g, :n]
            p = self.pos[l, b, g, :n]
        else:
            ps = s.page_size
            npg = (n + ps - 1) // ps
            pages = self.block_table_host[b, :npg].astype(np.int64)
            idx = torch.as_tensor(pages, device=self.K.device)
            k = self.K[l, idx, g].reshape(npg * ps, s.head_dim)[:n]
            v = self.V[l, idx, g].reshape(npg * ps, s.head_dim)[:n]
            p = self.pos[l, idx, g].reshape(npg * ps)[:n]
        return (k.view(torch.int16).cpu().numpy().view(np.uint16),
                v.view(torch.int16).cpu().numpy().view(np.uint16),
                p.cpu().numpy().astype(np.int32))

    def unit_stats(self, u: int):
        s = self.spec
        l, _, g = self.unit_index(u)
        h0, h1 = g * s.group, (g + 1) * s.group
        return self.q_mean[l, h0:h1], self.q_norm_mean[l, h0:h1], self.R[l, h0:h1]

    @property
    def lens_host(self):
        return self.lens.cpu().numpy()

    @property
    def t_host(self):
        return self.t.cpu().numpy()

    @property
    def block_table_host(self):
        return None if self.block_table is None else self.block_table.cpu().numpy()


def make_cache(spec: CacheSpec, seed: int, device="cpu", lens=None, t=None,
               layers: Optional[Sequence[int]] = None) -> Cache:
    """Draw a full cache for ``spec``.

    ``lens``/``t`` override the spec's per-sequence lengths/positions.
    Dense caches are ``[L][batch][Hkv][cap][d]``; paged caches are per-layer
    pools ``[L][pages][Hkv][page_size][d]`` reached through a block table
    ``[batch][max_pages]`` whose physical page order is a random permutation.
    """
    gen = torch.Generator().manual_seed(seed)
    dgen = torch.Generator(device=device).manual_seed(seed + 1) if str(device) != "cpu" else gen
    L, B, H, d = spec.n_layers, spec.batch, spec.n_kv_heads, spec.head_dim
    lens_r, t_r = resolve_lens_t(spec, gen)
    if lens is not None:
        lens_r = list(lens)
    if t is not None:
        t_r = list(t)
    elif spec.positions == "from_zero":
        t_r = list(lens_r)
    if len(lens_r) != spec.batch or len(t_r) != spec.batch:
        raise ValueError(f"{spec.name}: {len(lens_r)} lengths and {len(t_r)} query positions for a batch of "
                         f"{spec.batch}")
    maxlen = max(lens_r) if lens_r else 0
    omega = torch.as_tensor(rope_omega(d, spec.rope_base), device=device)
    wdtype = torch.float64  # keys drawn and rotated in fp64 on every device, then rounded RNE to bf16
    nan_bits = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16)

    if spec.page_size:
        ps = spec.page_size
        npg = [(n + ps - 1) // ps for n in lens_r]
        max_pages = max(1, (max(maxlen, spec.cap) + ps - 1) // ps)
        n_pages = max(1, sum(npg))
        perm = torch.randperm(n_pages, generator=gen).to(torch.int32)
        bt = torch.full((B, max_pages), -1, dtype=torch.int32)
        o = 0
        for s in range(B):
            bt[s, :npg[s]] = perm[o:o + npg[s]]
            o += npg[s]
        cap = max_pages * ps
        K = torch.empty((L, n_pages, H, ps, d), dtype=torch.bfloat16, device=device)
        V = torch.empty_like(K)
        P = torch.full((L, n_pages, H, ps), -1, dtype=torch.int32, device=device)
        K.fill_(nan_bits.item()); V.fill_(nan_bits.item())
        block_table = bt.to(device)
    else:
        cap = max(spec.cap, maxlen, 1)
        K = torch.empty((L, B, H, cap, d), dtype=torch.bfloat16, device=device)
        V = torch.empty_like(K)
        P = torch.full((L, B, H, cap), -1, dtype=torch.int32, device=device)
        K.fill_(nan_bits.item()); V.fill_(nan_bits.item())
        block_table = None
        n_pages = 0

    lens_dev = torch.as_tensor(lens_r, dtype=torch.int32)
    for l in range(L):
        centre = torch.randn((H, d), generator=dgen, device=device, dtype=wdtype)
        lo, hi = spec.key_sigma
        sigma = lo + (hi - lo) * torch.rand((H,), generator=dgen, device=device, dtype=wdtype)
        pos_l = _positions_for_layer(spec, gen, lens_r, t_r, cap if not spec.page_size else maxlen, device)
        for s in range(B):
            n = lens_r[s]
            if n == 0:
                continue
            noise = torch.randn((H, n, d), generator=dgen, device=device, dtype=wdtype)
            k_pre = centre[:, None, :] + sigma[:, None, None] * noise
            k_rot = _rotate(k_pre, pos_l[s, :, :n], omega, spec.layout).to(torch.bfloat16)
            v = torch.randn((H, n, d), generator=dgen, device=device, dtype=torch.float32).to(torch.bfloat16)
            p = pos_l[s, :, :n]
            if spec.page_size:
                ps = spec.page_size
                full = npg[s] * ps
                kk = torch.full((H, full, d), nan_bits.item(), dtype=torch.bfloat16, device=device)
                vv = kk.clone()
                pp = torch.full((H, full), -1, dtype=torch.int32, device=device)
                kk[:, :n] = k_rot; vv[:, :n] = v; pp[:, :n] = p
                pages = block_table[s, :npg[s]].long()
                K[l, pages] = kk.reshape(H, npg[s], ps, d).transpose(0, 1)
                V[l, pages] = vv.reshape(H, npg[s], ps, d).transpose(0, 1)
                P[l, pages] = pp.reshape(H, npg[s], ps).transpose(0, 1)
            else:
                K[l, s, :, :n] = k_rot
                V[l, s, :, :n] = v
                P[l, s] = pos_l[s]
    stats = make_stats(spec, seed)
    return Cache(spec, K, V, P, lens_dev.to(device), torch.as_tensor(t_r, dtype=torch.int32).to(device),
                 block_table, n_pages, cap, stats)


def replace(spec: CacheSpec, **kw) -> CacheSpec:
    return dataclasses.replace(spec, **kw)


def make_queries(n_layers: int, T: int, n_q_heads: int, head_dim: int, seed: int,
                 sigma=(0.05, 1.5), device="cpu") -> torch.Tensor:
    """Pre-RoPE query samples for calibration: bf16 [n_layers][T][n_q_heads][head_dim].

    Per (layer, head) a centre drawn N(0, 1) per dim and a spread drawn U[sigma]; every token
    is centre + spread * N(0, 1) per dim, so heads range from tightly concentrated to diffuse.
    One band of head 0 in every layer is all zero (the degenerate band).
    """
    gen = torch.Generator().manual_seed(seed * 104729 + 3)
    c = torch.randn((n_layers, 1, n_q_heads, head_dim), generator=gen)
    sp = sigma[0] + (sigma[1] - sigma[0]) * torch.rand((n_layers, 1, n_q_heads, 1), generator=gen)
    q = torch.empty((n_layers, T, n_q_heads, head_dim), dtype=torch.bfloat16)
    step = max(1, (1 << 24) // max(1, n_q_heads * head_dim))
    for l in range(n_layers):
        for t0 in range(0, T, step):
            t1 = min(T, t0 + step)
            z = torch.randn((t1 - t0, n_q_heads, head_dim), generator=gen)
            q[l, t0:t1] = (c[l] + sp[l] * z).to(torch.bfloat16)
    q[:, :, 0, 0] = 0
    q[:, :, 0, head_dim // 2] = 0
    q[:, :, 0, 1] = 0
    return q.to(device)
