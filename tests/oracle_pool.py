"""Process-pool helpers that run the fp64 oracle over whole full-size
workloads for the dense parity checks (test infrastructure only).

The pool uses the "spawn" start method: the tests that call it have already
initialised CUDA, and a process forked after that would hang. Each task gets
one kv group's slice of the inputs and of the selection, so the oracle sees a
problem with Hkv = 1 and returns that group's outputs.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np


def _prefill_group(args):
    """Oracle forward and backward of some query blocks of one kv group.

    args: (q [1][G][N][d], k, v [1][1][N][d], do [1][G][N][d] as storage-dtype
    CPU tensors; idx/cnt/logg of the group [1][1][T][k]; storage dtype; the
    query blocks ts). Returns o, lse, dq [G][N][d] / [G][N] (rows of ts),
    these blocks' contributions to dk, dv [N][d], and dlogg [T][k] (rows of
    ts), fp64, with the row term D of the backward taken on o rounded to the
    storage dtype, as the interface passes the stored output in.
    """
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):  # one BLAS thread per worker process
        return _prefill_group_1(args)


def _prefill_group_1(args):
    from gated_block_sparse_b200 import inputs
    from oracle import sas_oracle as O

    q, k, v, do, idx, cnt, logg, dtype, ts = args
    _, G, N, d = q.shape
    st = lambda rows: inputs.to_storage(rows, dtype).double().numpy()  # noqa: E731
    o = np.zeros((G, N, d))
    lse = np.zeros((G, N))
    dq = np.zeros((G, N, d))
    dk = np.zeros((N, d))
    dv = np.zeros((N, d))
    dlogg = np.zeros(idx.shape[2:])
    for t in ts:
        res = O.query_block(q, k, v, do, idx, cnt, logg, 0, 0, t, o_stored=st)
        rows = slice(t * 64, min(N, (t + 1) * 64))
        for j in range(G):
            o[j, rows] = res["o"][j]
            lse[j, rows] = res["lse"][j]
            dq[j, rows] = res["dq"][j]
        np.add.at(dk, res["pos"], res["dk"])
        np.add.at(dv, res["pos"], res["dv"])
        kk = int(cnt[0, 0, t])
        dlogg[t, :kk] = res["dlogg"]
    return o, lse, dq, dk, dv, dlogg


def prefill_all(q, k, v, do, idx, cnt, logg, dtype: str, workers: int | None = None):
    """Oracle outputs of a whole prefill workload (B = 1). Each task is one
    kv group and every `split`-th query block of it (interleaved, so tasks
    cost about the same); the tasks' dk/dv contributions are summed. Returns
    dict(o, lse, dq, dk, dv, dlogg) in the library's layouts, fp64."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    T = idx.shape[2]
    assert B == 1
    ncpu = workers or os.cpu_count() or 1
    split = max(1, min(T, -(-ncpu // Hkv)))
    tasks = []
    for r in range(Hkv):
        part = (q[:, r * G:(r + 1) * G].clone(), k[:, r:r + 1].clone(), v[:, r:r + 1].clone(),
                do[:, r * G:(r + 1) * G].clone(), np.ascontiguousarray(idx[:, r:r + 1]),
                np.ascontiguousarray(cnt[:, r:r + 1]), np.ascontiguousarray(logg[:, r:r + 1]),
                dtype)
        for j in range(split):
            tasks.append((r, part + (list(range(T - 1 - j, -1, -split)),)))
    n = min(len(tasks), ncpu)
    if n > 1:
        with mp.get_context("spawn").Pool(n) as pool:
            res = pool.map(_prefill_group, [a for _, a in tasks])
    else:
        res = [_prefill_group(a) for _, a in tasks]
    out = dict(o=np.zeros((1, Hq, N, d)), lse=np.zeros((1, Hq, N)), dq=np.zeros((1, Hq, N, d)),
               dk=np.zeros((1, Hkv, N, d)), dv=np.zeros((1, Hkv, N, d)),
               dlogg=np.zeros(idx.shape))
    for (r, _), (o, lse, dq, dk, dv, dl) in zip(tasks, res):
        out["o"][0, r * G:(r + 1) * G] += o
        out["lse"][0, r * G:(r + 1) * G] += lse
        out["dq"][0, r * G:(r + 1) * G] += dq
        out["dk"][0, r] += dk
        out["dv"][0, r] += dv
        out["dlogg"][0, r] += dl
    return out
