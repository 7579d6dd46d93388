"""Plain definitions of the recurrent layer on tiny inputs (test infrastructure only).

Nothing here follows the buffered algorithm of ``sketch_oracle.c``.  The state is
advanced one token at a time with explicit K x K transition matrices, and the
outputs are the definitions themselves:

* exact output of step t:  y_t = S_t^T q_t, S_t = M_t S_{t-1} + beta_t k_t v_t^T
  (read-after-update; the SketchSSM abstract's full-state baseline);
* sketch output: the flushed state S_f is only ever read through the projector
  P = Omega_r^T Omega_r onto the head's first r basis vectors (paper abstract:
  outputs for the basis vectors are precomputed at the state update), while the
  tokens since the flush stay exact:
      y_t = S_t^T q_t - S_f^T (I - P) Phi_t^T q_t,   Phi_t = M_t ... M_{f+1};
* the Mamba-2 closed form of the replay, with weights w_i = prod_{j>i} a_j.
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np


def transition(kind: str, a, k, beta) -> np.ndarray:
    """Explicit transition matrix M of one token."""
    K = k.shape[0]
    eye = np.eye(K)
    if kind == "mamba2":
        return float(a) * eye
    erase = eye - float(beta) * np.outer(k, k)
    if kind == "gdn":
        return float(a) * erase
    if kind == "kda":
        return np.diag(np.asarray(a, dtype=np.float64)) @ erase
    raise ValueError(kind)


def write_gain(kind: str, beta) -> float:
    return 1.0 if kind == "mamba2" else float(beta)


def run_row(kind: str, S0: np.ndarray, tokens: List[dict], rank: np.ndarray,
            omega: np.ndarray, G: int, Hqk: int, W: int) -> dict:
    """One batch row, every head, every step, by the definitions above.

    S0 [H][K][V]; tokens[t] holds this row's q, k [Hqk][K], v [H][V], a, beta.
    Returns y_exact [T][H][V], y_sketch [T][H][V], and the states / sketches at each
    flush (after steps W, 2W, ...): S_flush [F][H][K][V], Y_flush [F][H] (list of r x V).
    """
    S0 = np.asarray(S0, dtype=np.float64)
    H, K, V = S0.shape
    T = len(tokens)
    y_exact = np.zeros((T, H, V))
    y_sketch = np.zeros((T, H, V))
    n_flush = T // W
    S_flush = np.zeros((n_flush, H, K, V))
    Y_flush: List[List[Optional[np.ndarray]]] = [[None] * H for _ in range(n_flush)]
    for h in range(H):
        qh = h * Hqk // H
        g = h * G // H
        r = int(rank[h])
        P = None if r < 0 else omega[g, :r].T @ omega[g, :r]
        S = S0[h].copy()
        S_f = S.copy()
        Phi = np.eye(K)
        for t, tok in enumerate(tokens):
            q = np.asarray(tok["q"][qh], dtype=np.float64)
            k = np.asarray(tok["k"][qh], dtype=np.float64)
            v = np.asarray(tok["v"][h], dtype=np.float64)
            a = tok["a"][h]
            beta = None if tok.get("beta") is None else tok["beta"][h]
            M = transition(kind, a, k, beta)
            S = M @ S + write_gain(kind, beta) * np.outer(k, v)
            Phi = M @ Phi
            y_exact[t, h] = S.T @ q
            if P is None:
                y_sketch[t, h] = y_exact[t, h]
            else:
                y_sketch[t, h] = y_exact[t, h] - S_f.T @ ((np.eye(K) - P) @ (Phi.T @ q))
            if (t + 1) % W == 0:
                f = (t + 1) // W - 1
                S_flush[f, h] = S
                if P is not None:
                    Y_flush[f][h] = omega[g, :r] @ S
                S_f = S.copy()
                Phi = np.eye(K)
    return {"y_exact": y_exact, "y_sketch": y_sketch, "S_flush": S_flush, "Y_flush": Y_flush}


def mamba2_closed_form(S_f: np.ndarray, Y_h: Optional[np.ndarray], omega_r: Optional[np.ndarray],
                       q: np.ndarray, ks: np.ndarray, vs: np.ndarray, a_s: np.ndarray) -> np.ndarray:
    """Mamba-2 decode of one head in closed form.

    ks [n][K], vs [n][V], a_s [n] are the buffered tokens oldest first (the current
    token last).  y = decay_prod * read(q) + sum_i w_i (k_i . q) v_i with
    w_i = prod_{j > i} a_j and decay_prod = prod_j a_j; read() is S_f^T q for a dense
    head and Y^T (Omega_r q) for a sketch head.
    """
    n = ks.shape[0]
    y = np.zeros(vs.shape[1])
    for i in range(n):
        w = float(np.prod(a_s[i + 1:]))
        y += w * float(ks[i] @ q) * vs[i]
    decay_prod = float(np.prod(a_s))
    if Y_h is None:
        y += decay_prod * (S_f.T @ q)
    else:
        y += decay_prod * (Y_h.T @ (omega_r @ q))
    return y
