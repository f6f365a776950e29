"""Seeded synthetic inputs for the SAS gated block-sparse attention path.

This module is shared by the CUDA path's callers and by the fp64 oracle. It
only draws and plants data; it computes no score, gate, Top-K, softmax or
attention. Planting needs one direction per kv group (the normalised mean of
the group's query heads, or a random unit vector) and each block's key mean;
both are input construction, not the method.

Workloads follow the pages' settings: block size 64, GQA 32/8 heads, d = 128,
Top-K budgets of 1024/2048/4096 tokens (SAS close reading, liuzhao09.github.io,
section 3.1 and Fig. 7), with q, k, v, dO ~ N(0, 1).

Every value is drawn in fp64 with numpy's PCG64 and rounded once, round to
nearest even, to the storage dtype (bf16 or fp32). Both sides consume the same
stored bytes.

Planting (so that the block ranking near the Top-K boundary is decided by a
margin far above fp32 rounding):
  * prefill: per kv group r a random unit w_r; every query of the group gets
    + q_shift * w_r; every complete key block m has its own noise mean removed
    and a_m * w_r added, so its key mean is exactly a_m * w_r before rounding.
  * decode: per (sequence, kv group) u = normalised mean of the group's
    (rounded) query heads; each history block's key mean is moved along u to a
    target projection: 0.5 + 0.01 * rank for the planted high-relevance
    blocks, and min(natural projection, 0.4) for the others.
"""
from __future__ import annotations

import numpy as np
import torch

BLOCK = 64

# The five workloads. Shapes, budgets and dtypes are fixed; `seed` is
# 1000 * config number + attempt.
CONFIGS = {
    "c1": dict(kind="prefill", dtype="f32", B=1, Hq=2, Hkv=2, d=64, N=512, topk=2,
               plant="pm05", seed=1000),
    "c2": dict(kind="decode", dtype="bf16", B=1, Hq=32, Hkv=8, d=128, Lmax=65536,
               lens=(65536, 65536), topk=15, gated=1, planted=32, seed=2000),
    "c3": dict(kind="prefill", dtype="bf16", B=1, Hq=32, Hkv=8, d=128, N=16384, topk=31,
               plant="ramp", seed=3000),
    "c4": dict(kind="decode", dtype="bf16", B=8, Hq=32, Hkv=8, d=128, Lmax=131072,
               lens=(98304, 131072), topk=31, gated=1, planted=32, seed=4000),
    "c5": dict(kind="decode", dtype="bf16", B=1, Hq=32, Hkv=8, d=128, Lmax=524288,
               lens=(524288, 524288), topk=63, gated=1, planted=64, seed=5000),
}

DESCRIPTIONS = {
    "c1": "tiny prefill fwd+bwd fp32, MHA 2 heads, d=64, N=512, top-k 2",
    "c2": "decode bf16, GQA 32/8, d=128, batch 1, context 64K, top-k 15 (1024-token budget)",
    "c3": "prefill fwd+bwd bf16, GQA 32/8, d=128, N=16384, top-k 31 (2048-token budget)",
    "c4": "batched decode bf16, GQA 32/8, d=128, batch 8, ragged 96K-128K, top-k 31",
    "c5": "long decode bf16, GQA 32/8, d=128, batch 1, context 512K, top-k 63 (4096-token budget)",
}


def _rne_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Bit patterns (uint16) of fp64 values rounded to the nearest bf16, ties
    to even.

    Works on the fp64 bit pattern: bf16 keeps 7 of the 52 stored mantissa
    bits, so the rounding point is bit 45; the bf16 pattern is then the sign,
    the exponent re-biased from 1023 to 127 and the 7 kept mantissa bits.
    Inputs here are N(0,1)-sized, far from bf16 overflow; zeros (and values in
    the subnormal range) map to signed zero. Processed in chunks that stay in
    cache.
    """
    src = np.ascontiguousarray(x, dtype=np.float64).reshape(-1).view(np.int64)
    out = np.empty(src.shape, dtype=np.uint16)
    step = 1 << 18
    for i in range(0, src.size, step):
        b = src[i:i + step]
        r = (b + (((b >> 45) & 1) + ((1 << 44) - 1))) >> 45  # sign|exp11|mant7, rounded
        e8 = np.clip(((r >> 7) & 0x7FF) - (1023 - 127), 0, 255)
        out[i:i + step] = ((r >> 3) & 0x8000) | (e8 << 7) | ((r & 0x7F) * (e8 > 0))
    return out.reshape(np.shape(x))


def _rne_bf16_f64(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (ties to even), returned as fp64."""
    bits = _rne_bf16_bits(x).astype(np.uint32) << np.uint32(16)
    return bits.view(np.float32).astype(np.float64)


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round an fp64 array once to `dtype` ('bf16' or 'f32') as a CPU tensor."""
    if dtype == "bf16":
        bits = _rne_bf16_bits(x).view(np.int16)
        return torch.from_numpy(bits).view(torch.bfloat16)
    if dtype == "f32":
        return torch.from_numpy(np.asarray(x, dtype=np.float64).astype(np.float32))
    raise ValueError(f"unknown dtype {dtype!r}")


def _unit(rng: np.random.Generator, d: int) -> np.ndarray:
    w = rng.standard_normal(d)
    return w / np.linalg.norm(w)


def gen_prefill(B: int, Hq: int, Hkv: int, N: int, d: int, dtype: str, seed: int,
                plant: str | None = None, q_shift: float = 1.0) -> dict:
    """q, k, v, dO for one prefill/training pass, layout [B][H][N][d].

    plant=None: plain N(0,1). plant='ramp': block key means a_m = 0.045 * pi(m)
    (pi a seeded permutation per kv group). plant='pm05': a_m = +-0.5 (seeded
    sign) + 0.02 * pi(m). Planting touches only complete 64-key blocks.
    """
    assert Hq % Hkv == 0
    G = Hq // Hkv
    rng = np.random.Generator(np.random.PCG64(seed))
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    do = rng.standard_normal((B, Hq, N, d))
    nfull = N // BLOCK
    if plant is not None and nfull > 0:
        for b in range(B):
            for r in range(Hkv):
                w = _unit(rng, d)
                perm = rng.permutation(nfull).astype(np.float64)
                if plant == "ramp":
                    a = 0.045 * perm
                elif plant == "pm05":
                    sign = np.where(rng.random(nfull) < 0.5, -1.0, 1.0)
                    a = 0.5 * sign + 0.02 * perm
                else:
                    raise ValueError(f"unknown planting {plant!r}")
                q[b, r * G:(r + 1) * G] += q_shift * w
                kb = k[b, r, :nfull * BLOCK].reshape(nfull, BLOCK, d)
                kb -= kb.mean(axis=1, keepdims=True)
                kb += a[:, None, None] * w[None, None, :]
    return dict(q=to_storage(q, dtype), k=to_storage(k, dtype),
                v=to_storage(v, dtype), do=to_storage(do, dtype))


def gen_decode(B: int, Hq: int, Hkv: int, Lmax: int, d: int, lens, dtype: str, seed: int,
               planted: int | None = None) -> dict:
    """q [B][Hq][d], caches kc, vc [B][Hkv][Lmax][d] and lens [B] (int32).

    `lens` is a sequence of B lengths (1 <= n <= Lmax). With `planted`, each
    (sequence, kv group) gets that many high-relevance history blocks (see the
    module docstring); rows with fewer history blocks than `planted` plant all.

    Streams: numpy's SeedSequence(seed) spawns one child for q and one per
    (sequence, kv group) row, so rows are independent draws that threads fill
    in parallel (numpy's generators and array kernels release the GIL) with
    the same bytes whatever the thread count.
    """
    import concurrent.futures as cf
    import os

    assert Hq % Hkv == 0
    G = Hq // Hkv
    lens = np.asarray(lens, dtype=np.int64)
    assert lens.shape == (B,) and (lens >= 1).all() and (lens <= Lmax).all()
    children = np.random.SeedSequence(seed).spawn(1 + B * Hkv)
    q = to_storage(np.random.Generator(np.random.PCG64(children[0])).standard_normal((B, Hq, d)),
                   dtype)
    qr = q.double().numpy()
    st = torch.bfloat16 if dtype == "bf16" else torch.float32
    kc = torch.empty((B, Hkv, Lmax, d), dtype=st)
    vc = torch.empty((B, Hkv, Lmax, d), dtype=st)

    def row(b: int, r: int) -> None:
        rng = np.random.Generator(np.random.PCG64(children[1 + b * Hkv + r]))
        C = (int(lens[b]) - 1) // BLOCK  # complete history blocks before the current one
        ks = rng.standard_normal((Lmax, d))
        if planted and C > 0:
            qbar = qr[b, r * G:(r + 1) * G].mean(axis=0)
            u = qbar / np.linalg.norm(qbar)
            kb = ks[:C * BLOCK].reshape(C, BLOCK, d)
            proj = kb.mean(axis=1) @ u
            target = np.minimum(proj, 0.4)
            npl = min(planted, C)
            chosen = rng.choice(C, size=npl, replace=False)
            target[chosen] = 0.5 + 0.01 * rng.permutation(npl)
            kb += (target - proj)[:, None, None] * u[None, None, :]
        kc[b, r] = to_storage(ks, dtype)
        del ks
        vc[b, r] = to_storage(rng.standard_normal((Lmax, d)), dtype)

    rows = [(b, r) for b in range(B) for r in range(Hkv)]
    big = Lmax * d >= (1 << 20)
    workers = min(len(rows), os.cpu_count() or 1, 16) if big else 1
    if workers > 1:
        with cf.ThreadPoolExecutor(max_workers=workers) as ex:
            for f in [ex.submit(row, b, r) for b, r in rows]:
                f.result()
    else:
        for b, r in rows:
            row(b, r)
    return dict(q=q, kc=kc, vc=vc, lens=torch.from_numpy(lens.astype(np.int32)))


def ragged_lens(B: int, lo: int, hi: int, seed: int) -> list[int]:
    """B sequence lengths uniform in [lo, hi], seeded."""
    rng = np.random.Generator(np.random.PCG64(seed + 17))
    return [int(x) for x in rng.integers(lo, hi + 1, size=B)]


def gen_config(name: str, attempt: int = 0) -> dict:
    """Inputs of one of the five named workloads."""
    c = CONFIGS[name]
    seed = c["seed"] + attempt
    if c["kind"] == "prefill":
        return gen_prefill(c["B"], c["Hq"], c["Hkv"], c["N"], c["d"], c["dtype"], seed,
                           plant=c["plant"])
    lo, hi = c["lens"]
    lens = [lo] * c["B"] if lo == hi else ragged_lens(c["B"], lo, hi, seed)
    return gen_decode(c["B"], c["Hq"], c["Hkv"], c["Lmax"], c["d"], lens, c["dtype"], seed,
                      planted=c["planted"])
