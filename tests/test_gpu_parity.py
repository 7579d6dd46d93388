"""GPU (libsketchssm via its C ABI) against the fp64 oracle on the same seeded inputs.

Bar: max |gpu - oracle| / max |oracle| <= 1e-4 for y at every decode step and for
S and Y after every flush; the layout tables are compared bit for bit.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import synth
from gpu_util import parity_run

pytestmark = pytest.mark.gpu
DENSE = synth.DENSE


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_state_read_b200 import build
    build.build()


def small(cid, **over):
    return synth.config(cid).replace(**over)


# ----------------------------------------------------------------------------- layout

def layout_tables():
    out = []
    for cid in (0, 1, 3, 4):
        cfg = synth.config(cid)
        out.append((f"config{cid}", cfg, synth.layer_rank_table(cfg)))
    for m in (4, 6, 10, 21):
        cfg = synth.config(2, mean_rank=m, batch=64)
        t = synth.stack_rank_tables(cfg)
        for layer in (0, 13, 26):
            out.append((f"stack-r{m}-l{layer}", cfg, t[layer]))
    rng = np.random.default_rng(0)
    cfg = synth.config(1)
    for i in range(3):
        r = rng.integers(1, cfg.cap + 1, cfg.H).astype(np.int32)
        r[rng.random(cfg.H) < 0.3] = DENSE
        out.append((f"random{i}", cfg, r))
    out.append(("mamba2-per-head-qk", cfg.replace(Hqk=cfg.H), synth.layer_rank_table(cfg)))
    out.append(("all-dense", cfg, np.full(cfg.H, DENSE, np.int32)))
    out.append(("all-cap", cfg, np.full(cfg.H, cfg.cap, np.int32)))
    return out


def decode_geometry(cfg):
    """Item limits of the combine launch: heads per item and rows of one stage."""
    maxnh = min(32, cfg.H // cfg.G)
    rows = max(40 * 1024 // (4 * cfg.V), cfg.K + cfg.W, cfg.cap + cfg.W)
    return maxnh, rows


def item_cost(cfg, rank, heads, n):
    return sum(int(rank[h]) + n for h in heads)


def expected_work(rank, cfg):
    """Definition of the per-n work lists: dense heads first (head order), then per group
    the sketch heads packed greedily in head order while their rows (r + n) fit."""
    maxnh, budget = decode_geometry(cfg)
    H, G, Hg = cfg.H, cfg.G, cfg.H // cfg.G
    dense = [-h - 1 for h in range(H) if rank[h] == DENSE]
    out = {}
    for n in range(1, cfg.W + 1):
        items = list(dense)
        for g in range(G):
            cur = []
            for h in range(g * Hg, (g + 1) * Hg):
                if rank[h] <= 0:
                    continue
                if cur and (item_cost(cfg, rank, cur + [h], n) > budget or len(cur) == maxnh):
                    items.append(cur[0] * 64 + cur[-1] - cur[0] + 1)
                    cur = []
                cur.append(h)
            if cur:
                items.append(cur[0] * 64 + cur[-1] - cur[0] + 1)
        out[n] = items
    return out


@pytest.mark.parametrize("name,cfg,rank", layout_tables(), ids=[t[0] for t in layout_tables()])
def test_layout_bit_exact(name, cfg, rank):
    import rank_state_read_b200 as rs
    plan = rs.Plan(cfg.kind, batch=1, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K, value_dim=cfg.V,
                   window=cfg.W, groups=cfg.G, basis_rows=cfg.Rb, rank_cap=cfg.cap, rank=rank.tolist())
    off, rmax, rtot = oracle.layout(rank, cfg.G)
    assert plan.offsets == off.tolist()
    assert plan.rmax == rmax.tolist()
    assert plan.r_total == rtot
    assert plan.work == expected_work(rank, cfg)
    # every sketch head lands in exactly one item of each list, within the stage budget
    _, budget = decode_geometry(cfg)
    for n, items in plan.work.items():
        seen = []
        for e in items:
            if e < 0:
                continue
            hs = [h for h in range(e // 64, e // 64 + e % 64) if rank[h] > 0]
            assert item_cost(cfg, rank, hs, n) <= budget
            seen += hs
        assert sorted(seen) == [h for h in range(cfg.H) if rank[h] > 0]
    plan.close()


def test_layout_with_explicit_contiguous_group_table():
    """A group table equal to the contiguous layout is accepted and gives the same
    tables as NULL."""
    import rank_state_read_b200 as rs
    cfg = synth.config(1)
    rank = synth.layer_rank_table(cfg)
    kw = dict(batch=1, heads=cfg.H, qk_heads=cfg.Hqk, key_dim=cfg.K, value_dim=cfg.V, window=cfg.W,
              groups=cfg.G, basis_rows=cfg.Rb, rank_cap=cfg.cap, rank=rank.tolist())
    a = rs.Plan(cfg.kind, **kw)
    b = rs.Plan(cfg.kind, group=[h // (cfg.H // cfg.G) for h in range(cfg.H)], **kw)
    assert (a.offsets, a.rmax, a.r_total, a.work) == (b.offsets, b.rmax, b.r_total, b.work)
    a.close()
    b.close()


# ----------------------------------------------------------------------------- small, every row

def test_config0_full_trajectory():
    """Tiny Mamba-2 layer, all 64 steps (4 flushes), every element."""
    parity_run(synth.config(0), 64)


def test_config0_dense_read_trajectory():
    parity_run(synth.config(0), 40, dense=True)


@pytest.mark.parametrize("cid,B", [(1, 3), (3, 3), (4, 2)])
def test_layer_shapes_small_batch(cid, B):
    """The pages' layer shapes at a small ragged batch: 2 flushes plus 7 buffered steps."""
    parity_run(small(cid, B=B), 39)


@pytest.mark.parametrize("cid,B", [(1, 3), (3, 2), (4, 2)])
def test_dense_read_small_batch(cid, B):
    parity_run(small(cid, B=B), 20, dense=True)


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_all_heads_dense(kind):
    cid = {"mamba2": 1, "gdn": 3, "kda": 4}[kind]
    cfg = small(cid, B=2)
    parity_run(cfg, 18, rank=np.full(cfg.H, DENSE, np.int32))


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_all_heads_at_rank_cap(kind):
    cid = {"mamba2": 1, "gdn": 3, "kda": 4}[kind]
    cfg = small(cid, B=2)
    parity_run(cfg, 18, rank=np.full(cfg.H, cfg.cap, np.int32))


def test_rank_one_and_dense_mix():
    cfg = small(1, B=2)
    rank = np.ones(cfg.H, np.int32)
    rank[::5] = DENSE
    rank[:16] = DENSE            # group 0 has no sketch head at all
    parity_run(cfg, 18, rank=rank)


def test_partial_window_flushes():
    """Flushes after 5, 16 and 3 more buffered tokens (n < W, then a fresh window)."""
    parity_run(small(3, B=2), 30, flush_at=[5, 21, 24])


def test_per_head_qk_mamba2():
    """Mamba-2 with per-head q/k (Hqk = H): chains per head inside each group."""
    parity_run(small(1, B=2, Hqk=128), 18)


def test_shared_qk_gdn():
    """GDN with q/k shared by the heads of a group (Hqk = G)."""
    parity_run(small(3, B=2, Hqk=4), 18)


@pytest.mark.parametrize("V,W,H,G", [(16, 5, 8, 2), (48, 7, 64, 2), (256, 8, 4, 1), (128, 1, 32, 1)])
def test_other_shapes(V, W, H, G):
    """Value dims, odd windows, 32 heads per group (the largest item), W = 1."""
    cfg = small(3, B=2, V=V, W=W, H=H, G=G, Hqk=H, n_dense=1)
    parity_run(cfg, 2 * W + 3)


MAMBA2_SHAPES = [(16, 5, 8, 2, 2), (48, 7, 64, 2, 64), (256, 8, 4, 1, 1), (128, 1, 32, 1, 1),
                 (256, 4, 32, 1, 32), (80, 32, 32, 2, 2)]


@pytest.mark.parametrize("V,W,H,G,Hqk", MAMBA2_SHAPES)
def test_other_shapes_mamba2(V, W, H, G, Hqk):
    """Mamba-2 at other value dims, windows and group sizes (up to 32 heads and 256
    columns per group, the largest one-launch CTA), q/k shared by a group or per head."""
    cfg = small(1, B=3, V=V, W=W, H=H, G=G, Hqk=Hqk, n_dense=1)
    parity_run(cfg, 2 * W + 3)


@pytest.mark.parametrize("cid", [1, 3, 4])
def test_ring_reuse_moderate_batch(cid):
    """Enough batch rows that every persistent decode CTA walks several units through
    its stage ring (KDA's large dense items leave room for a one-stage ring)."""
    cfg = small(cid, B=96)
    parity_run(cfg, 18, rows=[0, 1, 47, 95])


def test_single_row_batch():
    parity_run(small(1, B=1), 17)


# ----------------------------------------------------------------------------- full size, every row

FULL = [(1, 20), (3, 18), (4, 17)]


@pytest.mark.parametrize("cid,T", FULL, ids=[f"config{c}" for c, _ in FULL])
def test_full_size_all_rows(cid, T):
    """The workloads at their full batch, in the bench's launch configuration, every
    batch row against the oracle (a flush of 16 tokens and the steps after it)."""
    parity_run(synth.config(cid), T, name=f"full-config{cid}")


@pytest.mark.parametrize("cid", [1, 3])
def test_full_size_dense_read_all_rows(cid):
    parity_run(synth.config(cid), 17, dense=True, name=f"full-dense-read-config{cid}")


def test_full_size_per_head_qk_mamba2_sampled_rows():
    """The Mamba-2 layer with q/k per head (the layer's secondary q/k layout)."""
    cfg = synth.config(1).replace(Hqk=128)
    parity_run(cfg, 17, rows=[0, 1, 77, 128, 255], name="full-config1-per-head-qk")


# ----------------------------------------------------------------------------- the 27-layer stack sweep

STACK_POINTS = [(m, B) for m in (4, 6, 10, 21) for B in (64, 256, 1024)]


def stack_layers(table):
    """The layer with the most dense heads and the one with the fewest (ties: first)."""
    nd = (table == DENSE).sum(axis=1)
    return int(np.argmax(nd)), int(np.argmin(nd))


@pytest.mark.parametrize("m,B", STACK_POINTS, ids=[f"r{m}-b{B}" for m, B in STACK_POINTS])
def test_stack_sweep_point(m, B):
    """Every point of the stack sweep (mean rank x batch): the most-dense and the
    least-dense layer of the point's rank tables, each with its own basis and inputs.
    Every row at batch 64 and 256; at batch 1024 a seeded sample of 64 rows (the
    others run on the GPU with states drawn on the device)."""
    cfg = synth.config(2, mean_rank=m, batch=B)
    table = synth.stack_rank_tables(cfg)
    one = cfg.replace(layers=1)
    rows = None
    if B > 256:
        rng = np.random.default_rng(1000 * m + B)
        rows = sorted({0, B - 1, *rng.choice(B, 62, replace=False).tolist()})
    for layer in sorted(set(stack_layers(table))):
        parity_run(one, 17, rank=table[layer], rows=rows, layer=layer,
                   init="numpy" if rows is None else "sampled", name=f"stack-r{m}-b{B}-layer{layer}")
