"""The decode loop around the prune: tri_append between prunes, a prune every C tokens, and the
pages past each pruned length returned to a free list and reused.

The page pool is tight, so freed pages come back into use. Before every prune the cache must
hold exactly the rows expected (the previous prune's output plus every appended row, bit for
bit); every prune is checked unit by unit against the fp64 oracle run on the rows it saw
(kept set up to threshold ties, compacted rows bit-exact, lengths).
"""
import numpy as np
import pytest
import torch

import tri_synth as ts
import gpu_util as gu
import oracle
from rope_aware_key_tri_b200 import tri

pytestmark = pytest.mark.gpu

L, HKV, G, D, BATCH, PS, B, C = 2, 2, 4, 64, 3, 16, 48, 32
MAX_PAGES = 8                 # capacity 128 slots per unit
N_PAGES = 22                  # tight: a sequence holds at most ceil((B + C) / PS) = 5 pages at a prune
PREFILL = (5, 37, 46)
STEPS = 5 * C


def _bits(x):
    return x.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class Pool:
    """The caller's side of a paged cache: pools, block table and a FIFO free list of pages."""

    def __init__(self, rng):
        self.K = torch.from_numpy(rng.integers(0, 1 << 16, (L, N_PAGES, HKV, PS, D), dtype=np.uint16)
                                  .view(np.int16)).view(torch.bfloat16).cuda()   # garbage, never read
        self.V = self.K.clone()
        self.P = torch.full((L, N_PAGES, HKV, PS), -7, dtype=torch.int32, device="cuda")
        self.bt = np.full((BATCH, MAX_PAGES), -1, dtype=np.int32)
        self.bt_dev = torch.from_numpy(self.bt).cuda()
        self.free = list(range(N_PAGES))
        self.reused = 0
        self.handed = set()

    def ensure(self, s, slot):
        j = slot // PS
        if self.bt[s, j] < 0:
            p = self.free.pop(0)
            if p in self.handed:
                self.reused += 1
            self.handed.add(p)
            self.bt[s, j] = p

    def reclaim(self, s, n):
        for j in range((n + PS - 1) // PS, MAX_PAGES):
            if self.bt[s, j] >= 0:
                self.free.append(int(self.bt[s, j]))
                self.bt[s, j] = -1

    def sync(self):
        self.bt_dev.copy_(torch.from_numpy(self.bt))

    def rows(self, l, s, g, n):
        slots = np.arange(n)
        pages = torch.from_numpy(self.bt[s, slots // PS].astype(np.int64)).cuda()
        offs = torch.from_numpy(slots % PS).cuda()
        return (_bits(self.K[l, pages, g, offs]), _bits(self.V[l, pages, g, offs]),
                self.P[l, pages, g, offs].cpu().numpy())


def test_decode_loop_append_prune_reclaim():
    rng = np.random.default_rng(11)
    spec = ts.CacheSpec(name="loop", head_dim=D, group=G, n_kv_heads=HKV, n_layers=L, batch=BATCH,
                        rope_base=1e4, budget=B, offsets=ts.pow2_offsets(10), positions="from_zero",
                        lens=(1,) * BATCH, key_sigma=(0.3, 0.3), page_size=PS)
    qm, qn, R, offsets = ts.make_stats(spec, 5)
    ctx = tri.TriContext(0)
    ctx.calibrate_load(L, HKV, G, D, spec.rope_base, spec.layout, qm, qn, R, offsets)
    pool = Pool(rng)
    lens = np.zeros(BATCH, dtype=np.int64)
    tpos = np.zeros(BATCH, dtype=np.int64)        # next position of each sequence
    expect = {(l, s, g): [np.zeros((0, D), np.uint16), np.zeros((0, D), np.uint16), np.zeros(0, np.int32)]
              for l in range(L) for s in range(BATCH) for g in range(HKV)}

    def draw():
        k = torch.from_numpy(rng.normal(0, 0.5, (L, BATCH, HKV, D)).astype(np.float32)).to(torch.bfloat16)
        v = torch.from_numpy(rng.normal(0, 1.0, (L, BATCH, HKV, D)).astype(np.float32)).to(torch.bfloat16)
        return k, v

    # prefill through the same entry point: sequence s takes part once its turn comes, so the
    # lengths end up ragged (PREFILL); a sequence outside its turn is refused by pointing its
    # slot at an unallocated page, which also exercises the refusal path
    for step in range(max(PREFILL)):
        active = [s for s in range(BATCH) if max(PREFILL) - PREFILL[s] <= step]
        for s in active:
            pool.ensure(s, int(lens[s]))
        pool.sync()
        k, v = draw()
        lens_dev = torch.from_numpy(lens.astype(np.int32)).cuda()
        pos_new = torch.from_numpy(tpos.astype(np.int32)).cuda()
        ctx.append(pool.K, pool.V, pool.P, lens_dev, pool.bt_dev, k.cuda(), v.cuda(), pos_new)
        st, code, unit = ctx.get_error()
        if len(active) < BATCH:
            assert st == tri.TRI_EDEVICE and code == 2, (st, code)  # TRI_DEV_BAD_PAGE
        else:
            assert st == tri.TRI_OK, (st, code, unit)
        new = lens_dev.cpu().numpy()
        for s in range(BATCH):
            if s in active:
                assert new[s] == lens[s] + 1
                for l in range(L):
                    for g in range(HKV):
                        e = expect[(l, s, g)]
                        e[0] = np.vstack([e[0], _bits(k[l, s, g])[None]])
                        e[1] = np.vstack([e[1], _bits(v[l, s, g])[None]])
                        e[2] = np.append(e[2], np.int32(tpos[s]))
                tpos[s] += 1
            else:
                assert new[s] == lens[s]
        lens = new.astype(np.int64)
    assert tuple(lens) == PREFILL

    prunes = 0
    for step in range(STEPS):
        for s in range(BATCH):
            pool.ensure(s, int(lens[s]))
        pool.sync()
        k, v = draw()
        lens_dev = torch.from_numpy(lens.astype(np.int32)).cuda()
        ctx.append(pool.K, pool.V, pool.P, lens_dev, pool.bt_dev, k.cuda(), v.cuda(),
                   torch.from_numpy(tpos.astype(np.int32)).cuda())
        assert ctx.get_error()[0] == tri.TRI_OK
        assert np.array_equal(lens_dev.cpu().numpy(), lens + 1)
        for l in range(L):
            for s in range(BATCH):
                for g in range(HKV):
                    e = expect[(l, s, g)]
                    e[0] = np.vstack([e[0], _bits(k[l, s, g])[None]])
                    e[1] = np.vstack([e[1], _bits(v[l, s, g])[None]])
                    e[2] = np.append(e[2], np.int32(tpos[s]))
        lens += 1
        tpos += 1
        if (step + 1) % C:
            continue
        # ---- a prune: the cache holds exactly what was appended since the last one ----------
        pre = {}
        for (l, s, g), e in expect.items():
            got = pool.rows(l, s, g, int(lens[s]))
            assert np.array_equal(got[0], e[0]) and np.array_equal(got[1], e[1]) and np.array_equal(got[2], e[2]), \
                f"step {step}: unit {(l, s, g)} does not hold the appended rows"
            pre[(l, s, g)] = got
        lens_dev = torch.from_numpy(lens.astype(np.int32)).cuda()
        t_dev = torch.from_numpy(tpos.astype(np.int32)).cuda()
        ctx.prune(pool.K, pool.V, pool.P, lens_dev, t_dev, B, block_table=pool.bt_dev)
        assert ctx.get_error()[0] == tri.TRI_OK
        new = lens_dev.cpu().numpy().astype(np.int64)
        assert np.array_equal(new, np.minimum(lens, B))
        for (l, s, g), (kb, vb, pb) in pre.items():
            n, m = int(lens[s]), int(new[s])
            out = pool.rows(l, s, g, m)
            if n > B:
                h0 = g * G
                orc = oracle.prune_unit(kb, vb, pb, int(tpos[s]), qm[l, h0:h0 + G], qn[l, h0:h0 + G],
                                        R[l, h0:h0 + G], offsets, spec.rope_base, B, spec.layout)
                kept = gu.kept_from_output(pb, out[2])
                gu.check_kept(kept, orc, B, f"prune {prunes} unit {(l, s, g)}")
                gu.check_compacted((kb, vb, pb), out, kept, f"prune {prunes} unit {(l, s, g)}")
            else:
                assert np.array_equal(out[0], kb[:m]) and np.array_equal(out[2], pb[:m])
            expect[(l, s, g)] = [out[0], out[1], out[2]]
        lens = new
        for s in range(BATCH):
            pool.reclaim(s, int(lens[s]))
        pool.sync()
        prunes += 1
    assert prunes == STEPS // C
    assert pool.reused > 0, "the tight pool never handed a freed page out again"
    ctx.close()


def test_append_refuses_full_sequences():
    spec = ts.CacheSpec(name="full", head_dim=128, group=2, n_kv_heads=1, n_layers=1, batch=2,
                        rope_base=1e4, budget=16, offsets=(1, 2), positions="from_zero", lens=(1, 1),
                        page_size=16)
    qm, qn, R, offsets = ts.make_stats(spec, 1)
    ctx = tri.TriContext(0)
    ctx.calibrate_load(1, 1, 2, 128, 1e4, spec.layout, qm, qn, R, offsets)
    K = torch.zeros((1, 2, 1, 16, 128), dtype=torch.bfloat16, device="cuda")
    V = torch.zeros_like(K)
    P = torch.zeros((1, 2, 1, 16), dtype=torch.int32, device="cuda")
    bt = torch.tensor([[0], [1]], dtype=torch.int32, device="cuda")   # one page each: capacity 16
    lens = torch.tensor([16, 3], dtype=torch.int32, device="cuda")     # sequence 0 is full
    kn = torch.ones((1, 2, 1, 128), dtype=torch.bfloat16, device="cuda")
    ctx.append(K, V, P, lens, bt, kn, kn, torch.tensor([16, 3], dtype=torch.int32, device="cuda"))
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == 1  # TRI_DEV_LEN_GT_CAP
    assert lens.cpu().tolist() == [16, 4]
    assert torch.all(K[0, 1, 0, 3] == 1) and int(P[0, 1, 0, 3]) == 3
    assert torch.all(K[0, 0] == 0)
    # host check: a dense cache (no block table) is rejected before anything is launched
    assert ctx.append(K, V, P, lens, None, kn, kn, lens, check=False) == tri.TRI_EINVAL
    ctx.close()


def test_append_advance_equals_append_then_position_update():
    """tri_append_advance: the same rows as tri_append, and the positions advanced by one for the
    sequences that accepted the token (a full sequence keeps its length and its position)."""
    spec = ts.CacheSpec(name="adv", head_dim=128, group=2, n_kv_heads=2, n_layers=2, batch=3,
                        rope_base=1e4, budget=16, offsets=(1, 2), positions="from_zero", lens=(1, 1, 1),
                        page_size=16)
    qm, qn, R, offsets = ts.make_stats(spec, 3)
    ctx = tri.TriContext(0)
    ctx.calibrate_load(2, 2, 2, 128, 1e4, spec.layout, qm, qn, R, offsets)
    gen = torch.Generator(device="cuda").manual_seed(5)
    steps = 5
    new_k = torch.randn((steps, 2, 3, 2, 128), generator=gen, device="cuda").to(torch.bfloat16)
    new_v = torch.randn((steps, 2, 3, 2, 128), generator=gen, device="cuda").to(torch.bfloat16)
    bt = torch.tensor([[0], [1], [2]], dtype=torch.int32, device="cuda")  # one page each: capacity 16

    def fresh():
        K = torch.zeros((2, 3, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
        # sequence 1 is two tokens from full, so it refuses the third step onwards
        return K, K.clone(), torch.full((2, 3, 2, 16), -1, dtype=torch.int32, device="cuda"), \
            torch.tensor([3, 14, 0], dtype=torch.int32, device="cuda"), \
            torch.tensor([100, 200, 300], dtype=torch.int32, device="cuda")

    K1, V1, P1, l1, t1 = fresh()
    for i in range(steps):
        before = l1.clone()
        ctx.append(K1, V1, P1, l1, bt, new_k[i], new_v[i], t1, check=False)
        t1.add_((l1 != before).to(torch.int32))  # the caller advances the accepted sequences
    K2, V2, P2, l2, t2 = fresh()
    for i in range(steps):
        ctx.append(K2, V2, P2, l2, bt, new_k[i], new_v[i], t2, check=False, advance=True)
    torch.cuda.synchronize()
    assert l1.cpu().tolist() == l2.cpu().tolist() == [8, 16, 5]
    assert t2.cpu().tolist() == [105, 202, 305]
    assert torch.equal(t1, t2)
    assert torch.equal(K1.view(torch.int16), K2.view(torch.int16))
    assert torch.equal(V1.view(torch.int16), V2.view(torch.int16))
    assert torch.equal(P1, P2)
    assert int(P2[1, 1, 1, 15]) == 201 and int(P2[0, 2, 0, 4]) == 304
    st, code, _ = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == 1  # TRI_DEV_LEN_GT_CAP (sequence 1)
    ctx.close()


def test_append_replays_from_a_cuda_graph():
    # the appends of a page span captured once and replayed give the same cache as the same
    # appends issued one by one
    spec = ts.CacheSpec(name="graph", head_dim=128, group=4, n_kv_heads=2, n_layers=2, batch=3,
                        rope_base=1e4, budget=16, offsets=(1, 2), positions="from_zero", lens=(1, 1, 1),
                        page_size=16)
    qm, qn, R, offsets = ts.make_stats(spec, 2)
    ctx = tri.TriContext(0)
    ctx.calibrate_load(2, 2, 4, 128, 1e4, spec.layout, qm, qn, R, offsets)
    steps = 16
    gen = torch.Generator(device="cuda").manual_seed(3)
    new_k = torch.randn((steps, 2, 3, 2, 128), generator=gen, device="cuda").to(torch.bfloat16)
    new_v = torch.randn((steps, 2, 3, 2, 128), generator=gen, device="cuda").to(torch.bfloat16)
    bt = torch.tensor([[0, 1], [2, 3], [4, 5]], dtype=torch.int32, device="cuda")

    def fresh():
        K = torch.zeros((2, 6, 2, 16, 128), dtype=torch.bfloat16, device="cuda")
        return K, K.clone(), torch.full((2, 6, 2, 16), -1, dtype=torch.int32, device="cuda"), \
            torch.tensor([16, 16, 16], dtype=torch.int32, device="cuda"), \
            torch.tensor([40, 50, 60], dtype=torch.int32, device="cuda")

    K1, V1, P1, l1, t1 = fresh()
    for i in range(steps):
        ctx.append(K1, V1, P1, l1, bt, new_k[i], new_v[i], t1)
        t1.add_(1)
    K2, V2, P2, l2, t2 = fresh()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
        for i in range(steps):
            ctx.append(K2, V2, P2, l2, bt, new_k[i], new_v[i], t2)
            t2.add_(1)
    torch.cuda.current_stream().wait_stream(side)
    assert l2.cpu().tolist() == [16, 16, 16]  # capturing ran nothing
    g.replay()
    torch.cuda.synchronize()
    assert ctx.get_error()[0] == tri.TRI_OK
    assert l1.cpu().tolist() == l2.cpu().tolist() == [32, 32, 32]
    assert torch.equal(K1.view(torch.int16), K2.view(torch.int16))
    assert torch.equal(V1.view(torch.int16), V2.view(torch.int16))
    assert torch.equal(P1, P2) and torch.equal(t1, t2)
    assert int(P1[0, 1, 0, 0]) == 40 and int(P1[1, 5, 1, 15]) == 75
    ctx.close()


@pytest.mark.parametrize("n_layers,n_kv,d", [(72, 8, 128), (5, 8, 64)])
def test_append_many_units_per_sequence(n_layers, n_kv, d):
    """Sequences with many (layer, KV head) units: 576 units per sequence take clusters of 8
    CTAs and two batches of loads per warp, 40 units take clusters of 3. Every unit of an
    accepted sequence receives its rows and position at slot lens[s] and nothing else changes;
    a sequence whose slot lands in an unallocated page is refused whole; lens (also lens_out)
    and the positions advance for the accepted ones only."""
    PS_, batch = 16, 4
    spec = ts.CacheSpec(name="wide", head_dim=d, group=2, n_kv_heads=n_kv, n_layers=n_layers, batch=batch,
                        rope_base=1e4, budget=16, offsets=(1, 2), positions="from_zero",
                        lens=(1,) * batch, page_size=PS_)
    qm, qn, R, offsets = ts.make_stats(spec, 4)
    ctx = tri.TriContext(0)
    ctx.calibrate_load(n_layers, n_kv, 2, d, 1e4, spec.layout, qm, qn, R, offsets)
    gen = torch.Generator(device="cuda").manual_seed(9)
    n_pages = 7
    K = torch.randn((n_layers, n_pages, n_kv, PS_, d), generator=gen, device="cuda").to(torch.bfloat16)
    V = torch.randn((n_layers, n_pages, n_kv, PS_, d), generator=gen, device="cuda").to(torch.bfloat16)
    P = torch.randint(0, 1000, (n_layers, n_pages, n_kv, PS_), generator=gen, device="cuda", dtype=torch.int32)
    new_k = torch.randn((n_layers, batch, n_kv, d), generator=gen, device="cuda").to(torch.bfloat16)
    new_v = torch.randn((n_layers, batch, n_kv, d), generator=gen, device="cuda").to(torch.bfloat16)
    # sequence 1's slot 16 is in its second page, which is not allocated: refused
    bt_h = [[0, 1], [2, -1], [3, 4], [5, 6]]
    lens_h = [5, 16, 31, 0]
    pos_h = [100, 200, 300, 400]
    bt = torch.tensor(bt_h, dtype=torch.int32, device="cuda")
    lens = torch.tensor(lens_h, dtype=torch.int32, device="cuda")
    pos = torch.tensor(pos_h, dtype=torch.int32, device="cuda")
    K_exp, V_exp, P_exp = K.clone(), V.clone(), P.clone()
    for s in (0, 2, 3):
        n = lens_h[s]
        page = bt_h[s][n // PS_]
        K_exp[:, page, :, n % PS_] = new_k[:, s]
        V_exp[:, page, :, n % PS_] = new_v[:, s]
        P_exp[:, page, :, n % PS_] = pos_h[s]
    ctx.append(K, V, P, lens, bt, new_k, new_v, pos, check=False, advance=True)
    torch.cuda.synchronize()
    st, code, unit = ctx.get_error()
    assert st == tri.TRI_EDEVICE and code == 2  # TRI_DEV_BAD_PAGE (sequence 1)
    assert unit == 1 * n_kv                       # reported as (layer 0, sequence 1, head 0)
    assert lens.cpu().tolist() == [6, 16, 32, 1]
    assert pos.cpu().tolist() == [101, 200, 301, 401]
    assert torch.equal(K.view(torch.int16), K_exp.view(torch.int16))
    assert torch.equal(V.view(torch.int16), V_exp.view(torch.int16))
    assert torch.equal(P, P_exp)
    ctx.close()
