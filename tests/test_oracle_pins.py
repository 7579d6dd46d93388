"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test names the fact it pins.  Together they are meant to fail on any plausible
slip in ``oracle/sketch_oracle.c`` (a dropped term, a wrong sign or index, a
transposed operand); ``test_mutations_are_caught`` checks that claim directly by
compiling altered copies of the oracle and running the brute-force pin on them.
"""
from __future__ import annotations

import os

import numpy as np
import pytest

import oracle
from oracle import brute
from oracle import build as obuild
import synth

DENSE = synth.DENSE


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))


def tiny_cfg(kind, *, H=4, G=2, Hqk=None, K=4, V=3, W=4, B=2, seed=77):
    Hqk = H if Hqk is None else Hqk
    return synth.Config(99, f"tiny-{kind}", kind, B=B, H=H, G=G, Hqk=Hqk, K=K, V=V, W=W,
                        Rb=K, cap=K, mean_rank=1, n_dense=0, steps=0, seed=seed)


def run_both(cfg, rank, T, *, omega=None, lib=None, inputs=None):
    """Oracle (sketch and dense modes) and brute force over T steps, every row."""
    omega = synth.basis_fp64(cfg) if omega is None else omega
    rows = list(range(cfg.B))
    S0 = synth.init_state(cfg, rows)
    steps = inputs if inputs is not None else [synth.step_inputs(cfg, t, rows) for t in range(T)]
    mk = lambda: oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W,
                                    G=cfg.G, rank=rank, omega=omega, S0=S0, lib=lib)
    sk, dn = mk(), mk()
    out_sk = list(oracle.trajectory(sk, steps))
    out_dn = list(oracle.trajectory(dn, steps, dense_all=True))
    bf = [brute.run_row(cfg.kind, S0[b], [{x: (None if s[x] is None else s[x][b]) for x in s}
                                          for s in steps], rank, omega, cfg.G, cfg.Hqk, cfg.W)
          for b in rows]
    return out_sk, out_dn, bf, sk


def check_against_brute(cfg, rank, T, **kw):
    out_sk, out_dn, bf, layer = run_both(cfg, rank, T, **kw)
    worst = 0.0
    f = 0
    for (ev_s, ev_d) in zip(out_sk, out_dn):
        if ev_s[0] == "decode":
            t = ev_s[1] - 1
            ys = np.stack([bf[b]["y_sketch"][t] for b in range(cfg.B)])
            yd = np.stack([bf[b]["y_exact"][t] for b in range(cfg.B)])
            worst = max(worst, rel(ev_s[2], ys), rel(ev_d[2], yd))
        elif ev_s[1] > 0:
            S = np.stack([bf[b]["S_flush"][f] for b in range(cfg.B)])
            worst = max(worst, rel(ev_s[2], S), rel(ev_d[2], S))
            for b in range(cfg.B):
                for h in range(cfg.H):
                    if rank[h] == DENSE:
                        continue
                    o = layer.off[h]
                    worst = max(worst, rel(ev_s[3][b, o:o + rank[h]], bf[b]["Y_flush"][f][h]))
            f += 1
    return worst


# --------------------------------------------------------------------------- layout

def layout_by_definition(rank, G):
    H = len(rank)
    off, acc = [], 0
    for h in range(H):
        off.append(acc)
        if rank[h] != DENSE:
            acc += int(rank[h])
    off.append(acc)
    rmax = [max([int(rank[h]) for h in range(H) if (h * G) // H == g and rank[h] != DENSE],
                default=0) for g in range(G)]
    return off, rmax, acc


def test_layout_golden_fixture(root):
    """Hand-derived layout of a small table (tests/golden/layout_small.txt)."""
    path = os.path.join(root, "tests", "golden", "layout_small.txt")
    fields = {}
    for line in open(path):
        line = line.split("#", 1)[0].strip()
        if line:
            key, val = line.split("=", 1)
            fields[key.strip()] = [int(x) for x in val.split()]
    G = fields["groups"][0]
    off, rmax, rtot = oracle.layout(np.array(fields["rank"], np.int32), G)
    assert off.tolist() == fields["off"]
    assert rmax.tolist() == fields["rmax"]
    assert rtot == fields["rtot"][0]


@pytest.mark.parametrize("seed", range(6))
def test_layout_matches_definition(seed):
    rng = np.random.default_rng(seed)
    H = int(rng.choice([1, 3, 8, 128, 3456]))
    G = int(rng.choice([g for g in (1, 2, 4, 8) if H % g == 0] or [1]))
    rank = rng.integers(1, 50, H).astype(np.int32)
    rank[rng.random(H) < 0.2] = DENSE
    off, rmax, rtot = oracle.layout(rank, G)
    e_off, e_rmax, e_rtot = layout_by_definition(rank, G)
    assert off.tolist() == e_off and rmax.tolist() == e_rmax and rtot == e_rtot


def test_layout_rejects_bad_rank():
    with pytest.raises(ValueError):
        oracle.layout(np.array([3, 0, 2], np.int32), 1)


# --------------------------------------------------------------------------- brute force

@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
@pytest.mark.parametrize("shared_qk", [False, True])
def test_tiny_brute_force(kind, shared_qk):
    """Buffered decode / flush equal the token-by-token definitions (read-after-update),
    dense and sketch heads, ranks 1..K, two full windows plus a ragged tail."""
    cfg = tiny_cfg(kind, Hqk=2 if shared_qk else None)
    rank = np.array([1, DENSE, 2, 4], np.int32)
    assert check_against_brute(cfg, rank, T=2 * cfg.W + 3) < 1e-12


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_full_size_head_brute_force(kind):
    """The same at the pages' head shape (K=128, V=80 / 128, W=16), ranks 1..49."""
    V = 80 if kind == "mamba2" else 128
    cfg = tiny_cfg(kind, H=4, G=2, K=128, V=V, W=16, B=1, seed=5)
    rank = np.array([49, 7, DENSE, 1], np.int32)
    assert check_against_brute(cfg, rank, T=20) < 1e-11


# --------------------------------------------------------------------------- invariants

@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_full_rank_sketch_is_exact(kind):
    """r = K with a full orthonormal (fp64) basis: the sketch read is the exact read."""
    V = 80 if kind == "mamba2" else 128
    cfg = tiny_cfg(kind, H=2, G=1, K=128, V=V, W=16, B=1, seed=11)
    rank = np.array([128, 128], np.int32)
    out_sk, out_dn, _, _ = run_both(cfg, rank, T=20)
    for es, ed in zip(out_sk, out_dn):
        if es[0] == "decode":
            assert rel(es[2], ed[2]) < 1e-12


def test_query_in_span_is_exact():
    """Mamba-2: a query inside span(omega_r) is read exactly at any rank r < K."""
    cfg = tiny_cfg("mamba2", H=2, G=1, K=128, V=80, W=16, B=1, seed=12)
    omega = synth.basis_fp64(cfg)
    r = 5
    rank = np.array([r, r], np.int32)
    rng = np.random.default_rng(3)
    steps = []
    for t in range(20):
        s = synth.step_inputs(cfg, t, [0])
        z = omega[0, :r].T @ rng.standard_normal(r)
        s["q"] = np.repeat((z / np.linalg.norm(z))[None, None, :], cfg.Hqk, axis=1)
        steps.append(s)
    out_sk, out_dn, _, _ = run_both(cfg, rank, 20, omega=omega, inputs=steps)
    for es, ed in zip(out_sk, out_dn):
        if es[0] == "decode":
            assert rel(es[2], ed[2]) < 1e-12


def test_sketch_prefix_property():
    """The sketch at rank r is the first r rows of the sketch at the full stored rank."""
    cfg = tiny_cfg("gdn", H=2, G=1, K=128, V=128, W=16, B=1, seed=13)
    omega = synth.basis_fp64(cfg)
    S0 = synth.init_state(cfg, [0])
    lo = oracle.OracleLayer("gdn", H=2, Hqk=2, K=128, V=128, W=16, G=1,
                            rank=np.array([3, 9], np.int32), omega=omega, S0=S0)
    hi = oracle.OracleLayer("gdn", H=2, Hqk=2, K=128, V=128, W=16, G=1,
                            rank=np.array([128, 128], np.int32), omega=omega, S0=S0)
    lo.flush(0)
    hi.flush(0)
    assert np.array_equal(lo.Y[0, 0:3], hi.Y[0, 0:3])
    assert np.array_equal(lo.Y[0, 3:12], hi.Y[0, 128:137])


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_flush_zero_and_one_token_flushes(kind):
    """flush(n=0) leaves S unchanged; one W-token flush equals W one-token flushes."""
    V = 80 if kind == "mamba2" else 128
    cfg = tiny_cfg(kind, H=2, G=1, K=128, V=V, W=16, B=2, seed=14)
    omega = synth.basis_fp64(cfg)
    S0 = synth.init_state(cfg, [0, 1])
    rank = np.array([4, DENSE], np.int32)
    mk = lambda: oracle.OracleLayer(kind, H=2, Hqk=2, K=128, V=V, W=16, G=1, rank=rank,
                                    omega=omega, S0=S0)
    A, Bl = mk(), mk()
    A.flush(0)
    assert np.array_equal(A.S, S0.astype(np.float64))
    steps = [synth.step_inputs(cfg, t, [0, 1]) for t in range(16)]
    for p, s in enumerate(steps):
        A.decode(p, s)
    A.flush(16)
    for s in steps:
        Bl.decode(0, s)
        Bl.flush(1)
    assert rel(A.S, Bl.S) < 1e-13
    assert rel(A.Y, Bl.Y) < 1e-13


def test_delta_rule_writes_value():
    """GDN with alpha = 1, beta = 1 and a unit key stores v exactly: S^T k = v after the
    update; KDA with a = 1 is the same operator."""
    cfg = tiny_cfg("gdn", H=1, G=1, K=128, V=128, W=16, B=1, seed=15)
    omega = synth.basis_fp64(cfg)
    S0 = synth.init_state(cfg, [0])
    s = synth.step_inputs(cfg, 0, [0])
    s["a"][:] = 1.0
    s["beta"][:] = 1.0
    k = s["k"][0, 0].astype(np.float64)
    k /= np.linalg.norm(k)            # unit in fp64 (the fp32 draw is unit only to 1e-8)
    s["k"] = k[None, None, :]
    g = oracle.OracleLayer("gdn", H=1, Hqk=1, K=128, V=128, W=16, G=1,
                           rank=np.array([DENSE], np.int32), omega=omega, S0=S0)
    g.decode(0, s)
    g.flush(1)
    assert rel(g.S[0, 0].T @ k, s["v"][0, 0]) < 1e-12
    s_k = dict(s)
    s_k["a"] = np.ones((1, 1, 128), np.float32)
    kd = oracle.OracleLayer("kda", H=1, Hqk=1, K=128, V=128, W=16, G=1,
                            rank=np.array([DENSE], np.int32), omega=omega, S0=S0)
    kd.decode(0, s_k)
    kd.flush(1)
    assert rel(kd.S, g.S) < 1e-14


def test_mamba2_closed_form_matches_chain():
    """Mamba-2 replay in closed form (w_i = prod_{j>i} a_j, decay_prod) equals the
    query-chain walk of the oracle, for dense and sketch heads."""
    cfg = synth.config(0).replace(B=2)
    rows = [0, 1]
    omega = synth.basis_fp64(cfg)
    rank = np.array([6, DENSE, 6, 6, 6, 6, 6, 6], np.int32)
    S0 = synth.init_state(cfg, rows)
    L = oracle.OracleLayer("mamba2", H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                           rank=rank, omega=omega, S0=S0)
    L.flush(0)
    hist = []
    for t in range(cfg.W + 5):
        pos = t % cfg.W
        s = synth.step_inputs(cfg, t, rows)
        if pos == 0:
            hist = []
            S_f, Y_f = L.S.copy(), L.Y.copy()
        hist.append(s)
        y = L.decode(pos, s)
        for b in rows:
            for h in range(cfg.H):
                ks = np.stack([x["k"][b, 0] for x in hist]).astype(np.float64)
                vs = np.stack([x["v"][b, h] for x in hist]).astype(np.float64)
                a_s = np.array([x["a"][b, h] for x in hist], np.float64)
                q = s["q"][b, 0].astype(np.float64)
                if rank[h] == DENSE:
                    e = brute.mamba2_closed_form(S_f[b, h], None, None, q, ks, vs, a_s)
                else:
                    o = L.off[h]
                    e = brute.mamba2_closed_form(None, Y_f[b, o:o + 6], omega[0, :6], q, ks, vs, a_s)
                assert rel(y[b, h], e) < 1e-12
        if pos == cfg.W - 1:
            L.flush(cfg.W)


# --------------------------------------------------------------------------- mutations

MUTATIONS = [
    # (name, original text, replacement, kind that must expose it)
    ("flush drops the decay",
     "Sh[kk * V + j] = a * Sh[kk * V + j] + ki[kk] * vi[j];",
     "Sh[kk * V + j] = Sh[kk * V + j] + ki[kk] * vi[j];", "mamba2"),
    ("flush erase sign",
     "a * (Sh[kk * V + j] - beta * ki[kk] * dv[j])",
     "a * (Sh[kk * V + j] + beta * ki[kk] * dv[j])", "gdn"),
    ("flush erase outside the decay",
     "a * (Sh[kk * V + j] - beta * ki[kk] * dv[j])",
     "(a * Sh[kk * V + j] - beta * ki[kk] * dv[j])", "kda"),
    ("flush projects with the wrong group",
     "omega + (g * d->Rb + m) * K;\n                double *Yr",
     "omega + (m) * K;\n                double *Yr", "mamba2"),
    ("chain drops the decay",
     "for (int64_t kk = 0; kk < K; ++kk) x[kk] = ai * x[kk];",
     "for (int64_t kk = 0; kk < K; ++kk) x[kk] = x[kk];", "mamba2"),
    ("chain erase sign",
     "x[kk] = ai * (x[kk] - bi * ki[kk] * s);",
     "x[kk] = ai * (x[kk] + bi * ki[kk] * s);", "gdn"),
    ("KDA transpose uses the undecayed query",
     "s2 += ki[kk] * xa[kk];",
     "s2 += ki[kk] * x[kk];", "kda"),
    ("replay drops beta",
     "yo[j] += bi * s * vi[j];",
     "yo[j] += s * vi[j];", "gdn"),
    ("read before update (current token skipped)",
     "for (int i = n - 1; i >= 0; --i) {",
     "for (int i = n - 2; i >= 0; --i) {", "mamba2"),
    ("sketch rows read at the wrong offset",
     "const double *Yr = Y + (b * rtot + off[h] + m) * V;",
     "const double *Yr = Y + (b * rtot + m) * V;", "mamba2"),
    ("sketch written at the wrong offset",
     "double *Yr = Y + (b * rtot + off[h] + m) * V;\n                for",
     "double *Yr = Y + (b * rtot + m) * V;\n                for", "gdn"),
    ("coefficients from the raw query",
     "c += om[kk] * x[kk];",
     "c += om[kk] * q[(b * d->Hqk + qh) * K + kk];", "gdn"),
]


@pytest.mark.parametrize("name,old,new,kind", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutations_are_caught(name, old, new, kind, tmp_path):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    out = str(tmp_path / "libmut.so")
    obuild.build(force=True, src=str(mutated), out=out)
    lib = oracle.load_library(out)
    cfg = tiny_cfg(kind, Hqk=2 if kind == "mamba2" else None)
    rank = np.array([1, DENSE, 2, 3], np.int32)
    assert check_against_brute(cfg, rank, T=2 * cfg.W + 3, lib=lib) > 1e-6


# --------------------------------------------------------------------------- standard step

def check_step_against_brute(cfg, T, lib=None):
    """The per-step recurrent decode (oracle.standard_step) against the token-by-token
    definition with explicit transition matrices (brute.run_row's exact read)."""
    rows = list(range(cfg.B))
    S = np.ascontiguousarray(synth.init_state(cfg, rows), dtype=np.float64)
    S0 = S.copy()
    steps = [synth.step_inputs(cfg, t, rows) for t in range(T)]
    rank = np.full(cfg.H, DENSE, np.int32)
    bf = [brute.run_row(cfg.kind, S0[b], [{x: (None if s[x] is None else s[x][b]) for x in s} for s in steps],
                        rank, synth.basis_fp64(cfg), cfg.G, cfg.Hqk, cfg.W) for b in rows]
    worst = 0.0
    for t, inp in enumerate(steps):
        y = oracle.standard_step(cfg.kind, S, inp, cfg.Hqk, lib=lib)
        worst = max(worst, rel(y, np.stack([bf[b]["y_exact"][t] for b in rows])))
    return worst


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
@pytest.mark.parametrize("shared_qk", [False, True])
def test_standard_step_brute_force(kind, shared_qk):
    """One token applied to the full state and read after the update, every step: equal
    to the explicit-matrix definition over two windows plus a ragged tail."""
    cfg = tiny_cfg(kind, Hqk=2 if shared_qk else None)
    assert check_step_against_brute(cfg, T=2 * cfg.W + 3) < 1e-12


def test_standard_step_full_head_shape():
    cfg = tiny_cfg("kda", H=2, G=1, K=128, V=128, W=16, B=1, seed=9)
    assert check_step_against_brute(cfg, T=5) < 1e-11


STEP_MUTATIONS = [
    ("step drops the decay",
     "Sh[kk * V + j] = at * Sh[kk * V + j] + kt[kk] * vt[j];",
     "Sh[kk * V + j] = Sh[kk * V + j] + kt[kk] * vt[j];", "mamba2"),
    ("step erase sign",
     "at * (Sh[kk * V + j] - bt * kt[kk] * e)",
     "at * (Sh[kk * V + j] + bt * kt[kk] * e)", "gdn"),
    ("step erase outside the decay",
     "at * (Sh[kk * V + j] - bt * kt[kk] * e)",
     "(at * Sh[kk * V + j] - bt * kt[kk] * e)", "kda"),
    ("step reads with the key",
     "s += Sh[kk * V + j] * qt[kk];",
     "s += Sh[kk * V + j] * kt[kk];", "gdn"),
]


@pytest.mark.parametrize("name,old,new,kind", STEP_MUTATIONS, ids=[m[0] for m in STEP_MUTATIONS])
def test_step_mutations_are_caught(name, old, new, kind, tmp_path):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    out = str(tmp_path / "libmut.so")
    obuild.build(force=True, src=str(mutated), out=out)
    lib = oracle.load_library(out)
    assert check_step_against_brute(tiny_cfg(kind, Hqk=2 if kind == "mamba2" else None), T=7, lib=lib) > 1e-6


# --------------------------------------------------------------------------- prefill handoff

def head_keys(cfg, k):
    """Token-major keys [B][T][Hqk][K] seen per state head: [B][T][H][K]."""
    return np.asarray(k, np.float64)[:, :, (np.arange(cfg.H) * cfg.Hqk) // cfg.H, :]


def prefilled(cfg, T, prompt=None, lib=None):
    rows = list(range(cfg.B))
    S = np.ascontiguousarray(synth.init_state(cfg, rows), dtype=np.float64)
    S0 = S.copy()
    prompt = synth.prompt_inputs(cfg, T, rows) if prompt is None else prompt
    oracle.prefill(cfg.kind, S, prompt, cfg.Hqk, lib=lib)
    return S0, S, prompt


def test_prefill_mamba2_closed_form():
    """Mamba-2 unrolls to S_T = (prod_t a_t) S_0 + sum_t (prod_{j>t} a_j) k_t v_t^T."""
    cfg = tiny_cfg("mamba2", Hqk=2)
    T = 2 * cfg.W + 3
    S0, S, p = prefilled(cfg, T)
    a = p["a"].astype(np.float64)
    w = np.ones_like(a)  # w[:, t] = prod_{j > t} a_j
    for t in range(T - 2, -1, -1):
        w[:, t] = w[:, t + 1] * a[:, t + 1]
    P = w[:, 0] * a[:, 0]
    exp = P[:, :, None, None] * S0 + np.einsum("bth,bthk,bthv->bhkv", w, head_keys(cfg, p["k"]),
                                               p["v"].astype(np.float64))
    assert rel(S, exp) < 1e-13


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_prefill_delta_rule_orthonormal_keys(kind):
    """No decay, beta = 1 and orthonormal keys: each token replaces the state's component
    along its key, so S_T = (I - sum_t k_t k_t^T) S_0 + sum_t k_t v_t^T."""
    cfg = tiny_cfg(kind, K=8, Hqk=2)
    T = 5
    p = synth.prompt_inputs(cfg, T, range(cfg.B))
    rng = np.random.default_rng(5)
    k = np.empty(p["k"].shape)
    for b in range(cfg.B):
        for qh in range(cfg.Hqk):
            Q, _ = np.linalg.qr(rng.standard_normal((cfg.K, cfg.K)))
            k[b, :, qh, :] = Q[:, :T].T
    p = dict(p, k=k, a=np.ones(p["a"].shape), beta=np.ones(p["beta"].shape))
    S0, S, _ = prefilled(cfg, T, prompt=p)
    kh = head_keys(cfg, k)
    proj = np.eye(cfg.K) - np.einsum("bthk,bthl->bhkl", kh, kh)
    exp = np.einsum("bhkl,bhlv->bhkv", proj, S0) + np.einsum("bthk,bthv->bhkv", kh, p["v"].astype(np.float64))
    assert rel(S, exp) < 1e-12


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_prefill_delta_rule_without_writes(kind):
    """beta = 0 leaves the decays alone: S_T = (prod_t a_t) S_0, per head (GDN) or per
    key row (KDA)."""
    cfg = tiny_cfg(kind)
    T = 7
    p = synth.prompt_inputs(cfg, T, range(cfg.B))
    p = dict(p, beta=np.zeros(p["beta"].shape))
    S0, S, _ = prefilled(cfg, T, prompt=p)
    P = np.prod(p["a"].astype(np.float64), axis=1)
    exp = (P[:, :, None, None] if kind == "gdn" else P[:, :, :, None]) * S0
    assert rel(S, exp) < 1e-13


def check_handoff_against_brute(cfg, rank, T, lib=None):
    """The handoff (prefill, then the n = 0 flush) against the explicit-matrix
    definition fed the same tokens one step at a time: brute.run_row's state and sketch
    at its last flush (T a multiple of W)."""
    rows = list(range(cfg.B))
    omega = synth.basis_fp64(cfg)
    S0 = synth.init_state(cfg, rows)
    p = synth.prompt_inputs(cfg, T, rows)
    layer = oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                               rank=rank, omega=omega, S0=S0, lib=lib)
    layer.prefill(p)
    steps = [{"q": p["k"][:, t], "k": p["k"][:, t], "v": p["v"][:, t], "a": p["a"][:, t],
              "beta": None if p["beta"] is None else p["beta"][:, t]} for t in range(T)]
    worst = 0.0
    for b in rows:
        bf = brute.run_row(cfg.kind, S0[b], [{x: (None if s[x] is None else s[x][b]) for x in s} for s in steps],
                           rank, omega, cfg.G, cfg.Hqk, cfg.W)
        worst = max(worst, rel(layer.S[b], bf["S_flush"][-1]))
        for h in range(cfg.H):
            if rank[h] != DENSE:
                o = layer.off[h]
                worst = max(worst, rel(layer.Y[b, o:o + rank[h]], bf["Y_flush"][-1][h]))
    return worst


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_prefill_handoff_brute_force(kind):
    """State and sketch after a prompt of two windows equal the token-by-token
    definition with explicit transition matrices."""
    cfg = tiny_cfg(kind, Hqk=2 if kind == "mamba2" else None)
    rank = np.array([1, DENSE, 2, 3], np.int32)
    assert check_handoff_against_brute(cfg, rank, T=2 * cfg.W) < 1e-12


def test_prefill_of_no_tokens_is_the_initial_flush():
    """T = 0: the state is unchanged and Y = Omega_r S_0 for every sketch head."""
    cfg = tiny_cfg("gdn")
    rank = np.array([1, DENSE, 2, 3], np.int32)
    omega = synth.basis_fp64(cfg)
    S0 = synth.init_state(cfg, range(cfg.B))
    layer = oracle.OracleLayer("gdn", H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                               rank=rank, omega=omega, S0=S0)
    layer.prefill(synth.prompt_inputs(cfg, 0, range(cfg.B)))
    assert np.array_equal(layer.S, S0.astype(np.float64))
    for h in range(cfg.H):
        if rank[h] != DENSE:
            g = h * cfg.G // cfg.H
            exp = np.einsum("mk,bkv->bmv", omega[g, :rank[h]], S0[:, h].astype(np.float64))
            assert rel(layer.Y[:, layer.off[h]:layer.off[h] + rank[h]], exp) < 1e-13


PREFILL_MUTATIONS = [
    ("prefill drops the decay",
     "St[r * V + c] = ap * St[r * V + c] + kp[r] * vp[c];",
     "St[r * V + c] = St[r * V + c] + kp[r] * vp[c];", "mamba2"),
    ("prefill erase sign",
     "ap * (St[r * V + c] - bp * kp[r] * ev[c])",
     "ap * (St[r * V + c] + bp * kp[r] * ev[c])", "gdn"),
    ("prefill tokens in reverse",
     "const int64_t bth = (b * T + t) * H + h;",
     "const int64_t bth = (b * T + (T - 1 - t)) * H + h;", "kda"),
    ("prefill key of the wrong q/k head",
     "const int64_t qh = (h * d->Hqk) / H;",
     "const int64_t qh = h % d->Hqk;", "mamba2"),
]


@pytest.mark.parametrize("name,old,new,kind", PREFILL_MUTATIONS, ids=[m[0] for m in PREFILL_MUTATIONS])
def test_prefill_mutations_are_caught(name, old, new, kind, tmp_path):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    out = str(tmp_path / "libmut.so")
    obuild.build(force=True, src=str(mutated), out=out)
    lib = oracle.load_library(out)
    cfg = tiny_cfg(kind, Hqk=2 if kind == "mamba2" else None)
    rank = np.array([1, DENSE, 2, 3], np.int32)
    assert check_handoff_against_brute(cfg, rank, T=2 * cfg.W, lib=lib) > 1e-6


# --------------------------------------------------------------------------- projected exact read

@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
def test_sketch_read_is_the_exact_read_of_the_projected_state(kind):
    """Right after a flush and at every later position of the window, a sketch head's
    output equals the exact output of the layer whose flushed state of that head is
    replaced by its projection P S_f (P = Omega_r^T Omega_r): the sketch only ever
    stands in for S_f, and the buffered tokens are replayed exactly.  Dense heads are
    read exactly in both."""
    cfg = tiny_cfg(kind, K=8, V=5, W=4, Hqk=2 if kind == "mamba2" else None)
    rank = np.array([3, DENSE, 1, 5], np.int32)
    rows = list(range(cfg.B))
    omega = synth.basis_fp64(cfg)
    S0 = synth.init_state(cfg, rows).astype(np.float64)
    Sp = S0.copy()
    for h in range(cfg.H):
        if rank[h] != DENSE:
            O = omega[h * cfg.G // cfg.H, :rank[h]]
            Sp[:, h] = np.einsum("kl,blv->bkv", O.T @ O, S0[:, h])
    mk = lambda S: oracle.OracleLayer(kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W, G=cfg.G,
                                      rank=rank, omega=omega, S0=S)
    sk, ex = mk(S0), mk(Sp)
    sk.flush(0)
    ex.flush(0)
    for t in range(cfg.W):
        inp = synth.step_inputs(cfg, t, rows)
        ys = sk.decode(t, inp)
        ye = ex.decode(t, inp, dense_all=True)
        assert rel(ys, ye) < 1e-12, t


@pytest.mark.parametrize("kind", ["mamba2", "gdn", "kda"])
@pytest.mark.parametrize("T", [3, 9])
def test_prefill_equals_the_buffered_update_path(kind, T):
    """The prompt path and the decode path update the state by the same recurrence: a
    prompt applied by prefill leaves the same state and sketch as its tokens appended one
    by one (decode, any query) with a flush after every W of them and one for the rest.
    Two separate routines of the oracle, so a mistake in either shows."""
    cfg = tiny_cfg(kind, Hqk=2 if kind == "mamba2" else None)
    rank = np.array([1, DENSE, 2, 3], np.int32)
    rows = list(range(cfg.B))
    omega = synth.basis_fp64(cfg)
    S0 = synth.init_state(cfg, rows)
    mk = lambda: oracle.OracleLayer(cfg.kind, H=cfg.H, Hqk=cfg.Hqk, K=cfg.K, V=cfg.V, W=cfg.W,
                                    G=cfg.G, rank=rank, omega=omega, S0=S0)
    pre, dec = mk(), mk()
    p = synth.prompt_inputs(cfg, T, rows)
    pre.prefill(p)
    pos = 0
    for t in range(T):
        tok = {"q": np.zeros((cfg.B, cfg.Hqk, cfg.K), np.float32), "k": p["k"][:, t], "v": p["v"][:, t],
               "a": p["a"][:, t], "beta": None if p["beta"] is None else p["beta"][:, t]}
        dec.decode(pos, tok)
        pos += 1
        if pos == cfg.W:
            dec.flush(pos)
            pos = 0
    dec.flush(pos)
    assert rel(dec.S, pre.S) < 1e-12
    assert rel(dec.Y, pre.Y) < 1e-12
