"""fp64 CPU oracle of SAS gated block-sparse causal attention.

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference arm may import this module. The library's kernels
never call it and share no code with it.

Plain, slow and written to be checked by eye against the pages:

* SAS close reading (liuzhao09.github.io, "SAS: learning context ranking
  under a finite attention budget"), section 2.1: the history is cut into
  contiguous blocks B_m of b tokens; s = R(q, {K_Bm}); I = TopK(s, k);
  S = B0 + the selected blocks; the current block B0 is always kept and is
  causally masked inside.
* same page, section 2.2: g_m = exp(s_m) / sum_l exp(s_l) over the C history
  blocks, g0 = 1, log g_m = s_m - LSE(s); o = softmax(q K_S^T + log g_S) V_S.
* SAS reproduction note (daiwk.github.io), core formula: the logit carries the
  1/sqrt(d) scale, o = softmax(q K_S^T / sqrt(d) + log g_S) V_S.
* SAS close reading, section 2.4: the backward pass recomputes the
  probabilities, forms the logit gradients from dO and sums them over each
  selected block into the block's log-gate gradient.
* SAS close reading, section 2.1 (Algorithm 2 as described there): at
  inference the continuous bias may be dropped and plain softmax attention
  runs over the Top-K blocks and the current block (`gated=0`).

Readings where the pages leave a step open:
* block size b = 64 (section 3.1); the selector is parameter-free:
  s_m = scale * qbar . kbar_m, kbar_m = mean of block m's 64 keys,
  qbar = mean of the kv group's query heads (and, in prefill, of the query
  block's tokens), scale = 1/sqrt(d);
* the gate softmax runs over all C causally visible complete history blocks;
* Top-K order is (score descending, block index ascending); the kept indices
  are listed in ascending block order, padded with -1; kk = min(k, C);
* prefill selects one block set per (sequence, kv group, 64-token query
  block); query block t sees history blocks 0..t-1 (C = t);
* decode: the query sits at position n-1, t = (n-1)//64, C = t and all n-64t
  tokens of the current block are visible.

Layouts: q/o/dO [B][Hq][N][d]; k/v [B][Hkv][N][d]; summaries [B][Hkv][nblk][d];
idx/logg/dlogg [B][Hkv][T][k] with T = ceil(N/64); cnt [B][Hkv][T];
lse [B][Hq][N]. All arithmetic in float64.
"""
from __future__ import annotations

import numpy as np

BLOCK = 64


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor: upcast its stored values
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# Block summaries (section 2.1: summaries compress each block's keys; the
# summary is the mean of the block's 64 keys).
# --------------------------------------------------------------------------
def block_summary(k, lens=None) -> np.ndarray:
    """kbar[b, r, m] = mean of the 64 keys of complete block m.

    With `lens`, blocks that are not complete within lens[b] are zero.
    """
    k = _f64(k)
    B, H, N, d = k.shape
    nblk = N // BLOCK
    out = np.zeros((B, H, nblk, d))
    for b in range(B):
        nb = nblk if lens is None else min(nblk, int(lens[b]) // BLOCK)
        for m in range(nb):
            out[b, :, m] = k[b, :, m * BLOCK:(m + 1) * BLOCK].mean(axis=1)
    return out


def round_bf16(x) -> np.ndarray:
    """The nearest bf16 value of each element (8 significant bits, ties to
    even), as float64: summaries stored in bf16 halve the bytes the
    long-context selection scans, and the selection then runs on these
    rounded values. Normal range only (summaries are means of the keys)."""
    x = _f64(x)
    m, e = np.frexp(x)  # x = m 2^e, 0.5 <= |m| < 1
    ulp = np.ldexp(1.0, e - 8)
    return np.round(x / ulp) * ulp  # numpy rounds halves to even


# --------------------------------------------------------------------------
# Selector score, normalised gate, Top-K (sections 2.1 and 2.2).
# --------------------------------------------------------------------------
def gate_and_topk(s: np.ndarray, topk: int):
    """For one row's scores s[0..C-1]: (idx ascending, log g of idx, log g of all).

    log g_m = s_m - LSE(s) with the max shift; Top-K keeps the kk = min(k, C)
    largest scores, ties to the lower block index.
    """
    C = s.shape[0]
    kk = min(topk, C)
    if C == 0:
        return np.zeros(0, dtype=np.int64), np.zeros(0), np.zeros(0)
    mx = s.max()
    lse = mx + np.log(np.exp(s - mx).sum())
    logg_all = s - lse
    order = np.lexsort((np.arange(C), -s))  # primary: -s ascending; then index
    chosen = np.sort(order[:kk])
    return chosen, logg_all[chosen], logg_all


def _pack_rows(B, Hkv, T, topk):
    idx = np.full((B, Hkv, T, topk), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv, T), dtype=np.int32)
    logg = np.zeros((B, Hkv, T, topk))
    return idx, cnt, logg


def select_prefill(q, ksum, Hkv: int, topk: int, scale: float | None = None):
    """Per (b, kv group r, query block t): scores, gate and Top-K.

    qbar = mean over the group's heads and the query block's tokens; C = t.
    Returns idx int32, cnt int32, logg (fp64), scores list-of-arrays.
    """
    q = _f64(q)
    ksum = _f64(ksum)
    B, Hq, N, d = q.shape
    G = Hq // Hkv
    T = -(-N // BLOCK)
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    idx, cnt, logg = _pack_rows(B, Hkv, T, topk)
    scores = {}
    for b in range(B):
        for r in range(Hkv):
            for t in range(T):
                rows = q[b, r * G:(r + 1) * G, t * BLOCK:min(N, (t + 1) * BLOCK)]
                qbar = rows.reshape(-1, d).mean(axis=0)
                C = t
                s = scale * (ksum[b, r, :C] @ qbar)
                chosen, lg, _ = gate_and_topk(s, topk)
                kk = chosen.shape[0]
                idx[b, r, t, :kk] = chosen
                cnt[b, r, t] = kk
                logg[b, r, t, :kk] = lg
                scores[(b, r, t)] = s
    return idx, cnt, logg, scores


def select_decode(q, ksum, lens, Hkv: int, topk: int, scale: float | None = None):
    """Per (b, kv group r): the decode query at position n-1, C = (n-1)//64.

    qbar = mean over the group's heads of q[b, h]. Returns idx [B][Hkv][k],
    cnt [B][Hkv], logg [B][Hkv][k] and the scores.
    """
    q = _f64(q)
    ksum = _f64(ksum)
    B, Hq, d = q.shape
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    idx = np.full((B, Hkv, topk), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv), dtype=np.int32)
    logg = np.zeros((B, Hkv, topk))
    scores = {}
    for b in range(B):
        C = (int(lens[b]) - 1) // BLOCK
        for r in range(Hkv):
            qbar = q[b, r * G:(r + 1) * G].mean(axis=0)
            s = scale * (ksum[b, r, :C] @ qbar)
            chosen, lg, _ = gate_and_topk(s, topk)
            kk = chosen.shape[0]
            idx[b, r, :kk] = chosen
            cnt[b, r] = kk
            logg[b, r, :kk] = lg
            scores[(b, r)] = s
    return idx, cnt, logg, scores


# --------------------------------------------------------------------------
# Gated sparse attention, forward (section 2.2; reproduction note's formula)
# and backward (section 2.4: recompute the probabilities, form the logit
# gradients from dO, sum them per selected block into d(log g)).
# --------------------------------------------------------------------------
def _token_set(t, N, sel, sel_logg):
    """Key positions and their bias for query block t: the selected history
    blocks (all 64 tokens, bias log g_m) followed by the current block
    (bias 0, g0 = 1). Returns positions, bias, and the current block's
    positions."""
    pos, bias = [], []
    for m, lg in zip(sel, sel_logg):
        pos.append(np.arange(m * BLOCK, (m + 1) * BLOCK))
        bias.append(np.full(BLOCK, float(lg)))
    cur = np.arange(t * BLOCK, min(N, (t + 1) * BLOCK))
    pos.append(cur)
    bias.append(np.zeros(cur.shape[0]))
    return np.concatenate(pos), np.concatenate(bias), cur


def _block_rows(qt, kS, vS, bias, cur, dot=None, scale=1.0, o_for_D=None):
    """Forward (and, with dot, backward) for the rows of one query block.

    qt [nr][d] are the rows i = cur[0..nr-1]; kS, vS [ns][d] the token set
    whose last len(cur) entries are the current block. Row i sees every
    history token and the current tokens j <= i (section 2.1, B0 causal).
    z = scale * q k^T + bias; p = softmax(z); o = p V; lse = log sum e^z.
    Backward of L = sum(dO * o): D_i = dO_i . o_i, dp = dO V^T,
    dz = p (dp - D), dq = scale dz K, dK = scale dz^T Q, dV = p^T dO.
    o_for_D, when given, is the output as the forward stored it (rounded to
    the storage dtype), or a function mapping the exact rows of o to their
    stored form; D then uses it, as the backward's interface defines D from
    the forward's output.
    """
    nr = qt.shape[0]
    nhist = kS.shape[0] - cur.shape[0]
    z = scale * (qt @ kS.T) + bias[None, :]
    causal = cur[None, :] <= cur[:, None]               # [row i][current j]
    z[:, nhist:] = np.where(causal, z[:, nhist:], -np.inf)
    mx = z.max(axis=1, keepdims=True)
    e = np.exp(z - mx)
    ssum = e.sum(axis=1, keepdims=True)
    p = e / ssum
    o = p @ vS
    lse = (mx + np.log(ssum))[:, 0]
    if dot is None:
        return o, lse
    if callable(o_for_D):
        o_for_D = o_for_D(o)
    D = (dot * (o if o_for_D is None else o_for_D)).sum(axis=1, keepdims=True)
    dp = dot @ vS.T
    dz = p * (dp - D)
    dq = scale * (dz @ kS)
    dkS = scale * (dz.T @ qt)
    dvS = p.T @ dot
    return o, lse, dq, dkS, dvS, dz


def _scale(d, scale):
    return 1.0 / np.sqrt(d) if scale is None else scale


def attn_fwd(q, k, v, idx, cnt, logg, scale: float | None = None):
    """o[b,h,i] = sum_j softmax_j(z_ij) v_j and lse[b,h,i] = log sum_j e^z_ij,
    z_ij = scale * q_i . k_j + log g of j's block (0 in the current block),
    over the selected blocks and the causal part of the current block."""
    q, k, v, logg = _f64(q), _f64(k), _f64(v), _f64(logg)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    T = -(-N // BLOCK)
    scale = _scale(d, scale)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            r = h // G
            for t in range(T):
                kk = int(cnt[b, r, t])
                pos, bias, cur = _token_set(t, N, idx[b, r, t, :kk], logg[b, r, t, :kk])
                o[b, h, cur], lse[b, h, cur] = _block_rows(
                    q[b, h, cur], k[b, r, pos], v[b, r, pos], bias, cur, scale=scale)
    return o, lse


def attn_bwd(q, k, v, do, idx, cnt, logg, scale: float | None = None, o_stored=None):
    """Gradients of L = sum(dO * o) with o from attn_fwd.

    dlogg[b, r, t, slot] = sum over the group's heads, the rows of query
    block t and the slot's 64 keys of the logit gradient dz (section 2.4).
    o_stored: optional forward output as stored (see _block_rows); the row
    term D_i = dO_i . o_i then uses it. Returns dq, dk, dv, dlogg.
    """
    if o_stored is not None and not callable(o_stored):
        o_stored = _f64(o_stored)
    q, k, v, do, logg = _f64(q), _f64(k), _f64(v), _f64(do), _f64(logg)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    T = -(-N // BLOCK)
    scale = _scale(d, scale)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dlogg = np.zeros(logg.shape)
    for b in range(B):
        for h in range(Hq):
            r = h // G
            for t in range(T):
                kk = int(cnt[b, r, t])
                pos, bias, cur = _token_set(t, N, idx[b, r, t, :kk], logg[b, r, t, :kk])
                _, _, dqt, dkS, dvS, dz = _block_rows(
                    q[b, h, cur], k[b, r, pos], v[b, r, pos], bias, cur,
                    dot=do[b, h, cur], scale=scale,
                    o_for_D=o_stored if (o_stored is None or callable(o_stored))
                    else o_stored[b, h, cur])
                dq[b, h, cur] = dqt
                np.add.at(dk[b, r], pos, dkS)
                np.add.at(dv[b, r], pos, dvS)
                for slot in range(kk):
                    dlogg[b, r, t, slot] += dz[:, slot * BLOCK:(slot + 1) * BLOCK].sum()
    return dq, dk, dv, dlogg


def query_block(q, k, v, do, idx, cnt, logg, b: int, r: int, t: int,
                scale: float | None = None, o_stored=None):
    """Forward and backward restricted to query block t of kv group r.

    The same definitions as attn_fwd / attn_bwd, for sampled checks of
    full-size workloads. Returns per head of the group: o, lse, dq (rows of
    block t), and dlogg[slot] summed over the group's heads, plus this
    block's dk/dv contributions {position array, dk rows, dv rows}.
    o_stored: optional function mapping exact output rows to their stored
    form, used for the row term D as in attn_bwd.
    """
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    scale = _scale(d, scale)
    kk = int(cnt[b, r, t])
    lg = _f64(logg[b, r, t, :kk])
    pos, bias, cur = _token_set(t, N, np.asarray(idx[b, r, t, :kk]), lg)
    kS, vS = _f64(k[b, r, pos]), _f64(v[b, r, pos])
    out = dict(o=[], lse=[], dq=[], dlogg=np.zeros(kk), pos=pos,
               dk=np.zeros_like(kS), dv=np.zeros_like(vS))
    for h in range(r * G, (r + 1) * G):
        o, lse, dq, dkS, dvS, dz = _block_rows(
            _f64(q[b, h, cur]), kS, vS, bias, cur, dot=_f64(do[b, h, cur]), scale=scale,
            o_for_D=o_stored)
        out["o"].append(o)
        out["lse"].append(lse)
        out["dq"].append(dq)
        out["dk"] += dkS
        out["dv"] += dvS
        for slot in range(kk):
            out["dlogg"][slot] += dz[:, slot * BLOCK:(slot + 1) * BLOCK].sum()
    return out


def key_block_grads(q, k, v, do, idx, cnt, logg, b: int, r: int, j: int,
                    scale: float | None = None, o_stored=None):
    """dk, dv of key block j of kv group r: the sum of the contributions of
    every query block that selected j, and of query block j itself (for
    which j is the current block)."""
    N = q.shape[2]
    T = -(-N // BLOCK)
    dk = np.zeros((BLOCK, q.shape[3]))
    dv = np.zeros((BLOCK, q.shape[3]))
    lo = j * BLOCK
    for t in range(T):
        kk = int(cnt[b, r, t])
        if t != j and j not in set(int(x) for x in idx[b, r, t, :kk]):
            continue
        res = query_block(q, k, v, do, idx, cnt, logg, b, r, t, scale, o_stored)
        hit = (res["pos"] >= lo) & (res["pos"] < lo + BLOCK)
        np.add.at(dk, res["pos"][hit] - lo, res["dk"][hit])
        np.add.at(dv, res["pos"][hit] - lo, res["dv"][hit])
    return dk, dv


# --------------------------------------------------------------------------
# Decode (section 2.1/2.4 serving: one query token per sequence, GQA groups
# share one block set).
# --------------------------------------------------------------------------
def decode(q, kc, vc, lens, ksum, Hkv: int, topk: int, gated: int = 1,
           scale: float | None = None):
    """One decode step. q [B][Hq][d]; kc, vc [B][Hkv][Lmax][d]; ksum the
    block summaries. Each (b, kv group) selects with select_decode; every
    head of the group attends over the selected blocks (bias log g when
    gated=1, none when gated=0) and the n-64t tokens of the current block.
    Returns o [B][Hq][d], idx [B][Hkv][k], cnt [B][Hkv], lse [B][Hq]."""
    q = _f64(q)
    B, Hq, d = q.shape
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    idx, cnt, logg, _ = select_decode(q, ksum, lens, Hkv, topk, scale)
    o, lse = decode_attend(q, kc, vc, lens, idx, cnt, logg, Hkv, gated, scale)
    return o, idx, cnt, lse


def decode_attend(q, kc, vc, lens, idx, cnt, logg, Hkv: int, gated: int = 1,
                  scale: float | None = None):
    """Decode attention for a given selection: every head of kv group r
    attends over the kept blocks idx[b, r, :cnt] (bias log g when gated=1,
    none when gated=0) and the n-64t tokens of the current block.
    Returns o [B][Hq][d], lse [B][Hq]."""
    q = _f64(q)
    logg = _f64(logg)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, Hq, d = q.shape
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    o = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b in range(B):
        n = int(lens[b])
        t = (n - 1) // BLOCK
        for r in range(Hkv):
            kk = int(cnt[b, r])
            pos, bias = [], []
            for slot in range(kk):
                m = int(idx[b, r, slot])
                pos.append(np.arange(m * BLOCK, (m + 1) * BLOCK))
                bias.append(np.full(BLOCK, logg[b, r, slot] if gated else 0.0))
            cur = np.arange(t * BLOCK, n)
            pos.append(cur)
            bias.append(np.zeros(cur.shape[0]))
            pos = np.concatenate(pos)
            bias = np.concatenate(bias)
            kr = _f64(kc[b, r][pos])
            vr = _f64(vc[b, r][pos])
            for h in range(r * G, (r + 1) * G):
                z = scale * (kr @ q[b, h]) + bias
                mx = z.max()
                e = np.exp(z - mx)
                o[b, h] = (e / e.sum()) @ vr
                lse[b, h] = mx + np.log(e.sum())
    return o, lse


# --------------------------------------------------------------------------
# Selector backward (section 2.3, eq. 8, sparse scope). The kept blocks'
# log-gate gradients reach every visible block's score through the shared
# normalisation log g = s - LSE(s); the parameter-free selector
# s_m = scale * qbar . kbar_m then carries the score gradient to the query
# and key means, and the means spread it over their rows.
# --------------------------------------------------------------------------
def select_backward(q, k, idx, cnt, dlogg, Hkv: int, scale: float | None = None,
                    return_ds: bool = False):
    """Gradient reaching q and k through the selector, given d(log g).

    For each (b, kv group r, query block t) with C = t visible history blocks,
    kept set I (the first cnt entries of idx) and g = softmax(s) over m < C:
        ds_m = dlogg[slot of m] * [m in I]  -  g_m * sum_{l in I} dlogg[slot of l]
    (eq. 8: for m outside I only the normalisation term remains). With
    s_m = scale * qbar_t . kbar_m:
        dqbar_t = scale * sum_m ds_m kbar_m,   dkbar_m += scale * ds_m qbar_t,
    qbar_t being the mean over the group's G heads and the n_t rows of block t,
    kbar_m the mean of block m's 64 keys; so each of those rows and heads gets
    dqbar_t / (G n_t) and each of block m's keys gets dkbar_m / 64.
    Returns (dq_sel [B][Hq][N][d], dk_sel [B][Hkv][N][d]) and, with
    return_ds, the ds rows {(b, r, t): ds[0..C-1]}. All in float64.
    """
    q, k, dlogg = _f64(q), _f64(k), _f64(dlogg)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, Hq, N, d = q.shape
    G = Hq // Hkv
    T = -(-N // BLOCK)
    scale = _scale(d, scale)
    ksum = block_summary(k)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    ds_rows = {}
    for b in range(B):
        for r in range(Hkv):
            dkbar = np.zeros((ksum.shape[2], d))
            for t in range(T):
                C = t
                if C == 0:
                    continue
                r0, r1 = t * BLOCK, min(N, (t + 1) * BLOCK)
                rows = q[b, r * G:(r + 1) * G, r0:r1]
                qbar = rows.reshape(-1, d).mean(axis=0)
                s = scale * (ksum[b, r, :C] @ qbar)
                g = np.exp(s - s.max())
                g = g / g.sum()
                kk = int(cnt[b, r, t])
                kept = [int(m) for m in idx[b, r, t, :kk]]
                total = sum(dlogg[b, r, t, j] for j in range(kk))
                ds = -g * total
                for j, m in enumerate(kept):
                    ds[m] += dlogg[b, r, t, j]
                ds_rows[(b, r, t)] = ds
                dqbar = scale * (ds @ ksum[b, r, :C])
                dq[b, r * G:(r + 1) * G, r0:r1] += dqbar / (G * (r1 - r0))
                dkbar[:C] += scale * np.outer(ds, qbar)
            for m in range(dkbar.shape[0]):
                dk[b, r, m * BLOCK:(m + 1) * BLOCK] += dkbar[m] / BLOCK
    if return_ds:
        return dq, dk, ds_rows
    return dq, dk


# --------------------------------------------------------------------------
# Per-token selection in prefill (section 2.4: the fused kernel masks the
# blocks a query did not select by that query's gate threshold, and skips a
# key tile that no query of the tile selected). Every query token i of kv
# group r selects its own blocks: qbar_i = mean of the group's G heads at
# token i, C_i = i // 64 visible history blocks, the same gate and Top-K
# rule as above. Layouts: idx/logg/dlogg [B][Hkv][N][k], cnt [B][Hkv][N].
# --------------------------------------------------------------------------
def select_prefill_tokens(q, ksum, Hkv: int, topk: int, scale: float | None = None):
    """Per (b, kv group r, query token i): scores, gate and Top-K over the
    C_i = i // 64 history blocks. Returns idx, cnt, logg and the scores
    {(b, r, i): s}."""
    q = _f64(q)
    ksum = _f64(ksum)
    B, Hq, N, d = q.shape
    G = Hq // Hkv
    scale = _scale(d, scale)
    idx = np.full((B, Hkv, N, topk), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv, N), dtype=np.int32)
    logg = np.zeros((B, Hkv, N, topk))
    scores = {}
    for b in range(B):
        for r in range(Hkv):
            for i in range(N):
                qbar = q[b, r * G:(r + 1) * G, i].mean(axis=0)
                C = i // BLOCK
                s = scale * (ksum[b, r, :C] @ qbar)
                chosen, lg, _ = gate_and_topk(s, topk)
                kk = chosen.shape[0]
                idx[b, r, i, :kk] = chosen
                cnt[b, r, i] = kk
                logg[b, r, i, :kk] = lg
                scores[(b, r, i)] = s
    return idx, cnt, logg, scores


def _token_keys(i, sel, sel_logg):
    """Key positions of query token i and their bias: each selected history
    block's 64 tokens (bias log g_m), then the current block's tokens up to
    and including i (bias 0, causal)."""
    pos, bias = [], []
    for m, lg in zip(sel, sel_logg):
        pos.append(np.arange(m * BLOCK, (m + 1) * BLOCK))
        bias.append(np.full(BLOCK, float(lg)))
    cur = np.arange((i // BLOCK) * BLOCK, i + 1)
    pos.append(cur)
    bias.append(np.zeros(cur.shape[0]))
    return np.concatenate(pos), np.concatenate(bias)


def _one_row(qi, kS, vS, bias, scale, dot=None, o_for_D=None):
    """One query row over its key set: z = scale k.q + bias, p = softmax(z),
    o = p V, lse = log sum e^z; with dot, the backward of L = dO . o:
    D = dO . o, dz = p (V dO - D), dq = scale dz K, dK = scale dz q^T,
    dV = p dO^T (o_for_D: the stored output used in D, if given)."""
    z = scale * (kS @ qi) + bias
    mx = z.max()
    e = np.exp(z - mx)
    ssum = e.sum()
    p = e / ssum
    o = p @ vS
    lse = mx + np.log(ssum)
    if dot is None:
        return o, lse
    D = dot @ (o if o_for_D is None else o_for_D)
    dz = p * (vS @ dot - D)
    return o, lse, scale * (dz @ kS), scale * np.outer(dz, qi), np.outer(p, dot), dz


def attn_fwd_tokens(q, k, v, idx, cnt, logg, scale: float | None = None):
    """o and lse of every head's rows, each query token over its own kept
    blocks (bias log g) and the causal part of its current block."""
    q, k, v, logg = _f64(q), _f64(k), _f64(v), _f64(logg)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    scale = _scale(d, scale)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            r = h // G
            for i in range(N):
                kk = int(cnt[b, r, i])
                pos, bias = _token_keys(i, idx[b, r, i, :kk], logg[b, r, i, :kk])
                o[b, h, i], lse[b, h, i] = _one_row(q[b, h, i], k[b, r, pos], v[b, r, pos],
                                                    bias, scale)
    return o, lse


def attn_bwd_tokens(q, k, v, do, idx, cnt, logg, scale: float | None = None, o_stored=None):
    """Gradients of L = sum(dO * o) with o from attn_fwd_tokens; dlogg[b, r,
    i, slot] sums dz over the group's heads and the slot's 64 keys of row i.
    o_stored: the forward output as stored, used in D (optional)."""
    q, k, v, do, logg = _f64(q), _f64(k), _f64(v), _f64(do), _f64(logg)
    if o_stored is not None:
        o_stored = _f64(o_stored)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    scale = _scale(d, scale)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dlogg = np.zeros(logg.shape)
    for b in range(B):
        for h in range(Hq):
            r = h // G
            for i in range(N):
                kk = int(cnt[b, r, i])
                pos, bias = _token_keys(i, idx[b, r, i, :kk], logg[b, r, i, :kk])
                _, _, dqi, dkS, dvS, dz = _one_row(
                    q[b, h, i], k[b, r, pos], v[b, r, pos], bias, scale, dot=do[b, h, i],
                    o_for_D=None if o_stored is None else o_stored[b, h, i])
                dq[b, h, i] = dqi
                np.add.at(dk[b, r], pos, dkS)
                np.add.at(dv[b, r], pos, dvS)
                for slot in range(kk):
                    dlogg[b, r, i, slot] += dz[slot * BLOCK:(slot + 1) * BLOCK].sum()
    return dq, dk, dv, dlogg


def select_backward_tokens(q, k, idx, cnt, dlogg, Hkv: int, scale: float | None = None):
    """Eq. 8 (sparse scope) for per-token selection: for each (b, r, token i)
    with C = i // 64, kept set I_i and g = softmax(s_i) over m < C,
        ds_m = dlogg[slot of m] [m in I_i] - g_m sum_{l in I_i} dlogg[slot of l];
    with s_m = scale qbar_i . kbar_m (qbar_i the mean of the group's G heads
    at token i), every head of the group gets scale sum_m ds_m kbar_m / G at
    token i, and block m's 64 keys get scale ds_m qbar_i / 64 each.
    Returns (dq_sel [B][Hq][N][d], dk_sel [B][Hkv][N][d]) in float64."""
    q, k, dlogg = _f64(q), _f64(k), _f64(dlogg)
    idx, cnt = np.asarray(idx), np.asarray(cnt)
    B, Hq, N, d = q.shape
    G = Hq // Hkv
    scale = _scale(d, scale)
    ksum = block_summary(k)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    for b in range(B):
        for r in range(Hkv):
            dkbar = np.zeros((ksum.shape[2], d))
            for i in range(N):
                C = i // BLOCK
                if C == 0:
                    continue
                qbar = q[b, r * G:(r + 1) * G, i].mean(axis=0)
                s = scale * (ksum[b, r, :C] @ qbar)
                g = np.exp(s - s.max())
                g = g / g.sum()
                kk = int(cnt[b, r, i])
                ds = -g * dlogg[b, r, i, :kk].sum()
                for j in range(kk):
                    ds[int(idx[b, r, i, j])] += dlogg[b, r, i, j]
                dq[b, r * G:(r + 1) * G, i] += scale * (ds @ ksum[b, r, :C]) / G
                dkbar[:C] += scale * np.outer(ds, qbar)
            for m in range(dkbar.shape[0]):
                dk[b, r, m * BLOCK:(m + 1) * BLOCK] += dkbar[m] / BLOCK
    return dq, dk
