"""Brute-force twin of the SAS oracle: dense, materialised, tiny sizes only.

TEST INFRASTRUCTURE (same rule as sas_oracle: only tests/, smoke() and the
bench's CPU arm may use it). Written separately from sas_oracle so that the
two can check each other:

* selection by enumeration: the chosen set is the k-subset of history blocks
  with the largest score sum, ties broken towards the lexicographically
  smallest index tuple (SAS close reading, liuzhao09.github.io, section 2.1:
  I = TopK(s, k); lower index wins a tie);
* attention on the full N x N logit matrix with an explicit visibility mask
  (selected blocks of the row's query block, plus the causal current block)
  and a dense bias matrix (log g of the key's block, 0 in the current block),
  as in the reproduction note's materialised check (daiwk.github.io,
  "reproduction boundary": the dense matrix validates selection and
  gradients);
* backward by the softmax Jacobian with the row term written as
  sum_j p_ij dp_ij, and d(log g) by summing dZ over each (query block,
  selected block) tile.
"""
from __future__ import annotations

import itertools

import numpy as np

BLOCK = 64


def topk_enumerate(s: np.ndarray, k: int) -> np.ndarray:
    """The k-subset of range(len(s)) maximising sum(s), lexicographically
    smallest on ties, returned ascending. Only for len(s) <= 10."""
    C = len(s)
    kk = min(k, C)
    best, best_sum = None, -np.inf
    for combo in itertools.combinations(range(C), kk):  # lexicographic order
        tot = float(sum(s[list(combo)])) if kk else 0.0
        if tot > best_sum:
            best, best_sum = combo, tot
    return np.array(best if best is not None else (), dtype=np.int64)


def masks(N: int, sel_rows: list[list[int]], logg_rows: list[list[float]]):
    """Dense visibility and bias for one (sequence, kv group).

    sel_rows[t] lists the history blocks kept for query block t and
    logg_rows[t] their log gates. Returns (visible [N][N] bool,
    bias [N][N], blockid [N][N] int: slot number for history keys, -1 for
    the current block, -2 where invisible).
    """
    vis = np.zeros((N, N), dtype=bool)
    bias = np.zeros((N, N))
    slot = np.full((N, N), -2, dtype=np.int64)
    for i in range(N):
        t = i // BLOCK
        for s_i, m in enumerate(sel_rows[t]):
            cols = slice(m * BLOCK, (m + 1) * BLOCK)
            vis[i, cols] = True
            bias[i, cols] = logg_rows[t][s_i]
            slot[i, cols] = s_i
        for j in range(t * BLOCK, i + 1):
            vis[i, j] = True
            slot[i, j] = -1
    return vis, bias, slot


def dense_forward_backward(q, k, v, do, idx, cnt, logg, scale=None):
    """Full materialised forward and backward for every head.

    q, do [B][Hq][N][d]; k, v [B][Hkv][N][d]; idx/cnt/logg as the oracle's.
    Returns o, lse, dq, dk, dv, dlogg (all fp64).
    """
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    logg = np.asarray(logg, dtype=np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    T = -(-N // BLOCK)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, N))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dlogg = np.zeros_like(logg)
    for b in range(B):
        for h in range(Hq):
            r = h // G
            sel = [[int(x) for x in idx[b, r, t, :cnt[b, r, t]]] for t in range(T)]
            lgs = [[float(x) for x in logg[b, r, t, :cnt[b, r, t]]] for t in range(T)]
            vis, bias, slot = masks(N, sel, lgs)
            Z = scale * q[b, h] @ k[b, r].T + bias
            Z[~vis] = -np.inf
            rowmax = Z.max(axis=1, keepdims=True)
            E = np.exp(Z - rowmax)
            P = E / E.sum(axis=1, keepdims=True)
            o[b, h] = P @ v[b, r]
            lse[b, h] = rowmax[:, 0] + np.log(E.sum(axis=1))
            dP = do[b, h] @ v[b, r].T
            dZ = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dq[b, h] = scale * dZ @ k[b, r]
            dk[b, r] += scale * dZ.T @ q[b, h]
            dv[b, r] += P.T @ do[b, h]
            for t in range(T):
                rows = slice(t * BLOCK, min(N, (t + 1) * BLOCK))
                for s_i in range(len(sel[t])):
                    dlogg[b, r, t, s_i] += dZ[rows][slot[rows] == s_i].sum()
    return o, lse, dq, dk, dv, dlogg
