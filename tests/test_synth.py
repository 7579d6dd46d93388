"""The seeded input generator against the shapes and counts printed on the pages."""
from __future__ import annotations

import os

import numpy as np
import pytest

import synth


def card(root):
    vals = {}
    for line in open(os.path.join(root, "tests", "golden", "nemotron_nano_card.txt")):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split("=", 1)
            vals[k.strip()] = [int(x) for x in v.split()]
    return vals


def test_layer_shape_matches_card(root):
    c = card(root)
    cfg = synth.config(1)
    assert cfg.H == c["state_heads_per_layer"][0]
    assert (cfg.K, cfg.V) == (c["key_dim"][0], c["value_dim"][0])
    assert cfg.G == c["basis_groups_per_layer"][0]
    assert cfg.W == c["window"][0]
    assert cfg.cap == c["rank_cap"][0]
    st = synth.config(2, mean_rank=6)
    assert st.layers == c["recurrent_layers"][0]
    assert (st.layers, st.G, st.Rb, st.K) == tuple(c["omega_shape"])


@pytest.mark.parametrize("m", [4, 6, 10, 21])
def test_stack_dense_and_sketch_counts(root, m):
    c = card(root)
    cfg = synth.config(2, mean_rank=m, batch=64)
    t = synth.stack_rank_tables(cfg)
    n_dense = int((t == synth.DENSE).sum())
    n_sketch = int((t != synth.DENSE).sum())
    assert [n_dense, n_sketch] == c[f"mean_rank_{m}"]
    sk = t[t != synth.DENSE]
    assert sk.min() >= 1 and sk.max() <= cfg.cap
    assert int(sk.sum()) == m * n_sketch


def test_layer_rank_tables():
    for cid in (0, 1, 3, 4):
        cfg = synth.config(cid)
        t = synth.layer_rank_table(cfg)
        assert t.shape == (cfg.H,) and t.dtype == np.int32
        assert int((t == synth.DENSE).sum()) == cfg.n_dense
        sk = t[t != synth.DENSE]
        assert int(sk.sum()) == cfg.mean_rank * sk.size
        assert sk.max() <= min(cfg.cap, cfg.Rb)


def test_basis_orthonormal_rows():
    cfg = synth.config(1)
    om = synth.basis_fp64(cfg)
    assert om.shape == (cfg.G, cfg.Rb, cfg.K)
    for g in range(cfg.G):
        assert np.allclose(om[g] @ om[g].T, np.eye(cfg.Rb), atol=1e-13)
    assert np.array_equal(synth.basis(cfg), om.astype(np.float32))


def test_step_inputs_distributions_and_row_independence():
    for cid in (1, 3, 4):
        cfg = synth.config(cid)
        s = synth.step_inputs(cfg, 5, [0, 1, 2, 3])
        assert np.allclose(np.linalg.norm(s["q"].astype(np.float64), axis=-1), 1, atol=1e-6)
        assert np.allclose(np.linalg.norm(s["k"].astype(np.float64), axis=-1), 1, atol=1e-6)
        if cfg.kda:
            assert s["a"].shape == (4, cfg.H, cfg.K)
            assert (s["a"] > np.float32(0.9)).all() and (s["a"] < np.float32(1.0)).all()
        else:
            assert s["a"].shape == (4, cfg.H)
            assert (s["a"] > 0).all() and (s["a"] < 1).all()
        assert (s["beta"] is None) == (cfg.kind == "mamba2")
        one = synth.step_inputs(cfg, 5, [2])
        for x in ("q", "k", "v", "a"):
            assert np.array_equal(one[x][0], s[x][2])


def test_prompt_rows_regenerate_alone_and_follow_the_step_distributions():
    """Every (row, token) of a prompt has its own stream: a subset of rows regenerates
    exactly; keys are unit vectors, decays lie in (0, 1), beta only for GDN / KDA."""
    for cid in (1, 3, 4):
        cfg = synth.config(cid)
        full = synth.prompt_inputs(cfg, 5, range(4))
        part = synth.prompt_inputs(cfg, 5, [2])
        for key in ("k", "v", "a"):
            assert np.array_equal(full[key][2:3], part[key])
        assert (full["beta"] is None) == (cfg.kind == "mamba2")
        assert np.allclose(np.linalg.norm(full["k"].astype(np.float64), axis=-1), 1.0, atol=1e-6)
        assert (full["a"] > 0).all() and (full["a"] < 1).all()
        assert full["k"].shape == (4, 5, cfg.Hqk, cfg.K) and full["v"].shape == (4, 5, cfg.H, cfg.V)
        # a prompt's tokens are not the decode steps' tokens
        step0 = synth.step_inputs(cfg, 0, range(4))
        assert not np.array_equal(full["v"][:, 0], step0["v"])
