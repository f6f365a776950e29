"""Pins of the fp64 oracle against things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle (a dropped bias, a
wrong sign or index, a missing causal mask, a transposed operand, a gate
normalised over the wrong set) fails at least one of them:

* dense equivalence: every history block selected and log g = 0 gives plain
  causal attention, checked against torch's scaled_dot_product_attention and
  its autograd in fp64 (a library routine);
* the brute-force twin (dense materialised masks, enumerated Top-K);
* torch autograd of an independently written dense masked formulation, for
  dq, dk, dv and d(log g);
* the K = 0 closed form (all scores 0: g = 1/C, the lowest indices win, the
  output is the gate-mass-weighted mean of V);
* central finite differences of d(log g), dq, dk, dv;
* the paper's eq. 5 form of the gate gradient (SAS close reading,
  liuzhao09.github.io, section 2.2): dL/dg_m = sum_{i in B_m} p~_i/g_m do.(v_i - o);
* gate invariants: sum g = 1, shift invariance (section 2.2), Top-K of s equals
  Top-K of g (order preservation, MSA notes, papercache, Top-K kernel section);
* per-token selection (section 2.4, the fused kernel's per-query threshold):
  reduction to the per-block oracle when every query block's rows are equal,
  the dense N x N masked logit matrix, and central finite differences.
"""
import numpy as np
import pytest
import torch

from gated_block_sparse_b200 import inputs
from oracle import brute
from oracle import sas_oracle as O

BLOCK = 64


def rnd(shape, seed):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape)


def full_selection(B, Hkv, N):
    """Every history block selected (k >= C), log g = 0."""
    T = -(-N // BLOCK)
    idx = np.full((B, Hkv, T, T), -1, dtype=np.int32)
    cnt = np.zeros((B, Hkv, T), dtype=np.int32)
    for t in range(T):
        idx[:, :, t, :t] = np.arange(t)
        cnt[:, :, t] = t
    return idx, cnt, np.zeros((B, Hkv, T, T))


# ---------------------------------------------------------------- inputs
def test_rne_bf16_matches_torch_on_fp32_values():
    x = rnd(100000, 1).astype(np.float32).astype(np.float64)  # fp32-exact values
    ours = inputs.to_storage(x, "bf16").float().numpy()
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours, ref)


def test_planting_moves_block_means():
    c = inputs.gen_prefill(1, 4, 2, 256, 16, "f32", seed=5, plant="ramp")
    k = c["k"].double().numpy()
    means = k[0, :, :256].reshape(2, 4, 64, 16).mean(axis=2)
    # each block's key mean is a multiple of one unit vector per kv group
    for r in range(2):
        norms = np.linalg.norm(means[r], axis=1)
        assert sorted(np.round(norms / 0.045).astype(int).tolist()) == [0, 1, 2, 3]


# ---------------------------------------------------------------- summaries
def test_block_summary_closed_form():
    B, H, N, d = 1, 2, 200, 3
    j = np.arange(N)[None, None, :, None]
    c = np.arange(d)[None, None, None, :]
    h = np.arange(H)[None, :, None, None]
    k = j + 1000.0 * c + 1e5 * h + np.zeros((B, H, N, d))
    ks = O.block_summary(k)
    assert ks.shape == (1, 2, 3, 3)  # the partial tail block has no summary
    for m in range(3):
        for cc in range(d):
            for hh in range(H):
                assert ks[0, hh, m, cc] == 64 * m + 31.5 + 1000 * cc + 1e5 * hh
    ks2 = O.block_summary(k, lens=[130])
    assert np.all(ks2[0, :, 2] == 0) and np.array_equal(ks2[0, :, :2], ks[0, :, :2])


# ---------------------------------------------------------------- gate / Top-K
def test_gate_invariants():
    s = rnd(37, 2)
    chosen, lg, lg_all = O.gate_and_topk(s, 5)
    assert abs(np.exp(lg_all).sum() - 1.0) < 1e-14          # sum_m g_m = 1
    c2, lg2, lg_all2 = O.gate_and_topk(s + 3.7, 5)          # shift invariance
    assert np.array_equal(chosen, c2) and np.allclose(lg_all, lg_all2, atol=1e-13)
    g = np.exp(lg_all)                                      # TopK(s) == TopK(g)
    assert set(np.argsort(-g)[:5].tolist()) == set(chosen.tolist())
    assert np.all(np.diff(chosen) > 0)                      # ascending order


@pytest.mark.parametrize("seed", range(40))
def test_topk_against_enumeration_with_ties(seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    C = int(rng.integers(0, 9))
    s = np.round(rng.standard_normal(C), 0)   # coarse values: many exact ties
    for k in range(0, 10):
        chosen, _, _ = O.gate_and_topk(s, k)
        assert chosen.tolist() == brute.topk_enumerate(s, k).tolist()


def test_topk_all_ties_takes_lowest_indices():
    chosen, lg, _ = O.gate_and_topk(np.zeros(9), 4)
    assert chosen.tolist() == [0, 1, 2, 3]
    assert np.allclose(lg, -np.log(9))


# ---------------------------------------------------------------- forward pins
def test_dense_equivalence_against_sdpa():
    B, Hq, Hkv, N, d = 1, 4, 2, 200, 16
    q, k, v = rnd((B, Hq, N, d), 3), rnd((B, Hkv, N, d), 4), rnd((B, Hkv, N, d), 5)
    idx, cnt, logg = full_selection(B, Hkv, N)
    o, lse = O.attn_fwd(q, k, v, idx, cnt, logg)
    G = Hq // Hkv
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(k).repeat_interleave(G, dim=1)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    assert np.abs(o - ref.numpy()).max() < 1e-12
    ref_lse = torch.logsumexp(
        (qt @ kt.transpose(-1, -2) / np.sqrt(d)).masked_fill(
            torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf")), dim=-1)
    assert np.abs(lse - ref_lse.numpy()).max() < 1e-12


def test_dense_equivalence_gradients_against_autograd():
    B, Hq, Hkv, N, d = 1, 4, 2, 160, 8
    q, k, v, do = (rnd((B, Hq, N, d), 6), rnd((B, Hkv, N, d), 7),
                   rnd((B, Hkv, N, d), 8), rnd((B, Hq, N, d), 9))
    idx, cnt, logg = full_selection(B, Hkv, N)
    dq, dk, dv, _ = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    G = Hq // Hkv
    qt = torch.from_numpy(q).requires_grad_()
    kt = torch.from_numpy(k).requires_grad_()
    vt = torch.from_numpy(v).requires_grad_()
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(G, dim=1), vt.repeat_interleave(G, dim=1), is_causal=True)
    (out * torch.from_numpy(do)).sum().backward()
    assert np.abs(dq - qt.grad.numpy()).max() < 1e-11
    assert np.abs(dk - kt.grad.numpy()).max() < 1e-11
    assert np.abs(dv - vt.grad.numpy()).max() < 1e-11


def _sparse_case(seed, N=256, d=16, Hq=4, Hkv=2, topk=2):
    q, k, v, do = (rnd((1, Hq, N, d), seed), rnd((1, Hkv, N, d), seed + 1),
                   rnd((1, Hkv, N, d), seed + 2), rnd((1, Hq, N, d), seed + 3))
    ks = O.block_summary(k)
    idx, cnt, logg, _ = O.select_prefill(q, ks, Hkv, topk)
    return q, k, v, do, idx, cnt, logg


@pytest.mark.parametrize("topk", [0, 1, 2, 3])
def test_against_bruteforce_twin(topk):
    q, k, v, do, idx, cnt, logg = _sparse_case(10 + topk, topk=topk)
    o, lse = O.attn_fwd(q, k, v, idx, cnt, logg)
    dq, dk, dv, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    bo, blse, bdq, bdk, bdv, bdlogg = brute.dense_forward_backward(q, k, v, do, idx, cnt, logg)
    for a, bb in ((o, bo), (lse, blse), (dq, bdq), (dk, bdk), (dv, bdv), (dlogg, bdlogg)):
        assert a.shape == bb.shape
        assert a.size == 0 or np.abs(a - bb).max() < 1e-11


def test_prefill_selection_against_enumeration():
    q, k, v, do, idx, cnt, logg = _sparse_case(20, N=512, topk=3)
    ks = O.block_summary(k)
    G = 2
    for r in range(2):
        for t in range(8):
            qbar = q[0, r * G:(r + 1) * G, t * 64:(t + 1) * 64].reshape(-1, 16).mean(axis=0)
            s = np.array([qbar @ ks[0, r, m] / 4.0 for m in range(t)])
            want = brute.topk_enumerate(s, 3)
            assert idx[0, r, t, :cnt[0, r, t]].tolist() == want.tolist()
            assert (idx[0, r, t, cnt[0, r, t]:] == -1).all()
            if t:
                g = np.exp(s) / np.exp(s).sum()
                assert np.allclose(logg[0, r, t, :cnt[0, r, t]], np.log(g[want]), atol=1e-13)


def test_prefill_query_pooling_closed_form():
    """The selector's query mean, pinned by construction rather than by
    re-slicing: q is zero except one token of one head, and every key of
    block m equals (m + 1) e_{m mod d}. Then qbar of row (r, t) is that
    token's vector / (G n_t) for the group holding the head and the block
    holding the token (n_t = the block's token count, 58 for the ragged last
    block here), and zero elsewhere, so every score has a closed form: a slip
    in the head range, the token range or the divisor changes some score."""
    B, Hq, Hkv, N, d = 1, 6, 3, 250, 4  # G = 2; T = 4 blocks, the last one 58 tokens
    G, T = Hq // Hkv, 4
    k = np.zeros((B, Hkv, N, d))
    for m in range(T):
        k[0, :, m * 64:min(N, (m + 1) * 64), m % d] = m + 1.0
    ks = O.block_summary(k)
    for h, i0, j, c in ((3, 200, 1, 5.0), (4, 249, 2, -3.0), (0, 64, 0, 2.0), (5, 130, 3, 7.0)):
        q = np.zeros((B, Hq, N, d))
        q[0, h, i0, j] = c
        _, _, _, scores = O.select_prefill(q, ks, Hkv, 2)
        t0, r0 = i0 // 64, h // G
        n_t0 = min(64, N - 64 * t0)
        for (b, r, t), srow in scores.items():
            assert len(srow) == t
            for m in range(t):
                want = 0.0
                if r == r0 and t == t0 and m % d == j:
                    want = (c / (G * n_t0)) * (m + 1.0) / np.sqrt(d)
                assert abs(srow[m] - want) < 1e-15, (h, i0, r, t, m, srow[m], want)


def test_decode_query_pooling_closed_form():
    """Decode: q nonzero in one head only; qbar = that head's vector / G for
    its group and zero for the others (closed-form scores as above)."""
    B, Hq, Hkv, L, d = 2, 8, 2, 512, 4  # G = 4
    G = Hq // Hkv
    kc = np.zeros((B, Hkv, L, d))
    for m in range(L // 64):
        kc[:, :, m * 64:(m + 1) * 64, m % d] = m + 1.0
    ks = O.block_summary(kc)
    lens = [512, 300]
    for b0, h, j, c in ((0, 5, 2, 4.0), (1, 2, 3, -1.5)):
        q = np.zeros((B, Hq, d))
        q[b0, h, j] = c
        _, _, _, scores = O.select_decode(q, ks, lens, Hkv, 3)
        for (b, r), srow in scores.items():
            C = (lens[b] - 1) // 64
            assert len(srow) == C
            for m in range(C):
                want = (c / G) * (m + 1.0) / np.sqrt(d) if (b == b0 and r == h // G
                                                             and m % d == j) else 0.0
                assert abs(srow[m] - want) < 1e-15


def _dense_torch_loss(q, k, v, do, idx, cnt, logg_t, scale):
    """Independent dense formulation in torch ops (mask + bias from a block
    map), differentiated by autograd; logg_t is a leaf [B][Hkv][T][k]."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    T = logg_t.shape[2]
    loss = 0.0
    for b in range(B):
        for h in range(Hq):
            r = h // G
            Z = scale * q[b, h] @ k[b, r].T
            bias = torch.zeros(N, N, dtype=torch.float64)
            allowed = torch.zeros(N, N, dtype=torch.bool)
            rows = torch.arange(N)
            for t in range(T):
                rs = slice(t * 64, min(N, (t + 1) * 64))
                for s_i in range(int(cnt[b, r, t])):
                    m = int(idx[b, r, t, s_i])
                    cs = slice(m * 64, (m + 1) * 64)
                    allowed[rs, cs] = True
                    bias = bias.index_put(
                        (rows[rs].repeat_interleave(64), torch.arange(m * 64, m * 64 + 64).repeat(rs.stop - rs.start)),
                        logg_t[b, r, t, s_i].expand((rs.stop - rs.start) * 64))
                allowed[rs, t * 64:min(N, (t + 1) * 64)] |= torch.ones(
                    rs.stop - rs.start, min(N, (t + 1) * 64) - t * 64, dtype=torch.bool).tril()
            Z = (Z + bias).masked_fill(~allowed, float("-inf"))
            o = torch.softmax(Z, dim=-1) @ v[b, r]
            loss = loss + (o * do[b, h]).sum()
    return loss


def test_gradients_against_autograd_sparse():
    q, k, v, do, idx, cnt, logg = _sparse_case(30, N=192, d=8, topk=1)
    dq, dk, dv, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    qt, kt, vt = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    lt = torch.from_numpy(logg).requires_grad_()
    loss = _dense_torch_loss(qt, kt, vt, torch.from_numpy(do), idx, cnt, lt, 1 / np.sqrt(8))
    loss.backward()
    assert np.abs(dq - qt.grad.numpy()).max() < 1e-11
    assert np.abs(dk - kt.grad.numpy()).max() < 1e-11
    assert np.abs(dv - vt.grad.numpy()).max() < 1e-11
    assert np.abs(dlogg - lt.grad.numpy()).max() < 1e-11


def test_k_zero_closed_form():
    """K = 0: every score is 0, g_m = 1/C, the lowest kk indices are kept, and
    o_i = [sum_{m in I} sum_{j in B_m} g_m v_j + sum_{j in B_t, j <= i} v_j]
          / [64 kk / C + (i - 64t + 1)]."""
    B, Hq, Hkv, N, d, topk = 1, 4, 2, 448, 16, 3
    q = rnd((B, Hq, N, d), 40)
    k = np.zeros((B, Hkv, N, d))
    v = rnd((B, Hkv, N, d), 41)
    idx, cnt, logg, _ = O.select_prefill(q, O.block_summary(k), Hkv, topk)
    o, _ = O.attn_fwd(q, k, v, idx, cnt, logg)
    for t in range(7):
        kk = min(topk, t)
        assert idx[0, 0, t, :kk].tolist() == list(range(kk))
        for i in range(t * 64, (t + 1) * 64):
            for h in range(Hq):
                r = h // 2
                num = v[0, r, t * 64:i + 1].sum(axis=0)
                den = i - 64 * t + 1
                for m in range(kk):
                    num = num + v[0, r, m * 64:(m + 1) * 64].sum(axis=0) / t
                    den += 64.0 / t
                assert np.abs(o[0, h, i] - num / den).max() < 1e-12


def test_k_zero_arbitrary_gates_weighted_mean():
    """K = 0 with arbitrary log g: history tokens weigh e^{log g_m}, current
    tokens weigh 1."""
    B, Hq, Hkv, N, d = 1, 2, 1, 256, 8
    q = rnd((B, Hq, N, d), 50)
    k = np.zeros((B, Hkv, N, d))
    v = rnd((B, Hkv, N, d), 51)
    T = 4
    idx = np.full((1, 1, T, 2), -1, dtype=np.int32)
    cnt = np.zeros((1, 1, T), dtype=np.int32)
    logg = np.zeros((1, 1, T, 2))
    idx[0, 0, 3] = [0, 2]
    cnt[0, 0, 3] = 2
    logg[0, 0, 3] = [-0.3, -2.1]
    idx[0, 0, 2, 0] = 1
    cnt[0, 0, 2] = 1
    logg[0, 0, 2, 0] = 0.7
    o, _ = O.attn_fwd(q, k, v, idx, cnt, logg)
    i = 3 * 64 + 10
    w0, w2 = np.exp(-0.3), np.exp(-2.1)
    num = w0 * v[0, 0, 0:64].sum(0) + w2 * v[0, 0, 128:192].sum(0) + v[0, 0, 192:i + 1].sum(0)
    den = 64 * w0 + 64 * w2 + 11
    assert np.abs(o[0, 1, i] - num / den).max() < 1e-12
    i = 2 * 64 + 63
    num = np.exp(0.7) * v[0, 0, 64:128].sum(0) + v[0, 0, 128:192].sum(0)
    assert np.abs(o[0, 0, i] - num / (64 * np.exp(0.7) + 64)).max() < 1e-12


# ---------------------------------------------------------------- backward pins
def _loss(q, k, v, do, idx, cnt, logg):
    o, _ = O.attn_fwd(q, k, v, idx, cnt, logg)
    return (o * do).sum()


def test_dlogg_central_finite_differences():
    q, k, v, do, idx, cnt, logg = _sparse_case(60, N=256, d=8, topk=2)
    _, _, _, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    h = 1e-5
    for (r, t, s) in [(0, 2, 0), (0, 3, 1), (1, 3, 0), (1, 2, 1), (0, 1, 0)]:
        lp, lm = logg.copy(), logg.copy()
        lp[0, r, t, s] += h
        lm[0, r, t, s] -= h
        fd = (_loss(q, k, v, do, idx, cnt, lp) - _loss(q, k, v, do, idx, cnt, lm)) / (2 * h)
        assert abs(fd - dlogg[0, r, t, s]) <= 1e-7 * max(1.0, abs(fd))


def test_qkv_central_finite_differences():
    q, k, v, do, idx, cnt, logg = _sparse_case(70, N=192, d=8, topk=1)
    dq, dk, dv, _ = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    h = 1e-5
    probes = [("q", dq, (0, 1, 150, 3)), ("q", dq, (0, 3, 70, 0)),
              ("k", dk, (0, 0, 10, 5)), ("k", dk, (0, 1, 130, 2)),
              ("v", dv, (0, 1, 64, 7)), ("v", dv, (0, 0, 191, 1))]
    for name, grad, ix in probes:
        args = dict(q=q, k=k, v=v)
        xp, xm = args[name].copy(), args[name].copy()
        xp[ix] += h
        xm[ix] -= h
        lp = _loss(**{**args, name: xp}, do=do, idx=idx, cnt=cnt, logg=logg)
        lm = _loss(**{**args, name: xm}, do=do, idx=idx, cnt=cnt, logg=logg)
        fd = (lp - lm) / (2 * h)
        assert abs(fd - grad[ix]) <= 1e-7 * max(1.0, abs(fd)), (name, ix, fd, grad[ix])


def test_dlogg_equals_eq5_form():
    """dL/dlog g_m = g_m dL/dg_m = sum_{i in B_m} p~_i do.(v_i - o) (eq. 5),
    summed over the query block's rows and the group's heads."""
    q, k, v, do, idx, cnt, logg = _sparse_case(80, N=320, d=8, topk=2)
    o, lse = O.attn_fwd(q, k, v, idx, cnt, logg)
    _, _, _, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    d = 8
    for r in range(2):
        for t in range(5):
            for s in range(int(cnt[0, r, t])):
                m = int(idx[0, r, t, s])
                tot = 0.0
                for h in (2 * r, 2 * r + 1):
                    for i in range(t * 64, (t + 1) * 64):
                        for jj in range(m * 64, (m + 1) * 64):
                            z = q[0, h, i] @ k[0, r, jj] / np.sqrt(d) + logg[0, r, t, s]
                            p_soft = np.exp(z - lse[0, h, i])
                            tot += p_soft * (do[0, h, i] @ (v[0, r, jj] - o[0, h, i]))
                assert abs(tot - dlogg[0, r, t, s]) < 1e-11


def test_row_gradients_sum_to_zero():
    """Each row's logit gradients sum to 0, so sum_slots dlogg[t] equals minus
    the current-block part of the dz sum over the block's rows and heads."""
    q, k, v, do, idx, cnt, logg = _sparse_case(90, N=256, d=16, topk=2)
    _, _, _, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    for r in range(2):
        for t in range(1, 4):
            cur_sum = 0.0
            for h in (2 * r, 2 * r + 1):
                kk = int(cnt[0, r, t])
                pos, bias, cur = O._token_set(t, 256, idx[0, r, t, :kk], logg[0, r, t, :kk])
                _, _, _, _, _, dz = O._block_rows(q[0, h, cur], k[0, r, pos], v[0, r, pos], bias,
                                                  cur, dot=do[0, h, cur], scale=0.25)
                cur_sum += dz[:, kk * 64:].sum()
            assert abs(dlogg[0, r, t].sum() + cur_sum) < 1e-12


def test_query_block_and_key_block_helpers():
    q, k, v, do, idx, cnt, logg = _sparse_case(95, N=320, d=8, topk=2)
    o, lse = O.attn_fwd(q, k, v, idx, cnt, logg)
    dq, dk, dv, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    res = O.query_block(q, k, v, do, idx, cnt, logg, 0, 1, 4)
    for j, h in enumerate((2, 3)):
        assert np.abs(res["o"][j] - o[0, h, 256:320]).max() < 1e-13
        assert np.abs(res["dq"][j] - dq[0, h, 256:320]).max() < 1e-13
    assert np.abs(res["dlogg"] - dlogg[0, 1, 4, :2]).max() < 1e-13
    for j in range(5):
        gk, gv = O.key_block_grads(q, k, v, do, idx, cnt, logg, 0, 0, j)
        assert np.abs(gk - dk[0, 0, j * 64:(j + 1) * 64]).max() < 1e-12
        assert np.abs(gv - dv[0, 0, j * 64:(j + 1) * 64]).max() < 1e-12


# ---------------------------------------------------------------- decode pins
@pytest.mark.parametrize("gated", [1, 0])
def test_decode_against_sdpa_mask(gated):
    """Decode = one query at n-1 over the kept blocks and the whole current
    block; checked with torch SDPA given a float mask (-inf / log g / 0)."""
    B, Hq, Hkv, L, d, topk = 2, 4, 2, 640, 16, 3
    lens = [600, 130]
    q = rnd((B, Hq, d), 100)
    kc, vc = rnd((B, Hkv, L, d), 101), rnd((B, Hkv, L, d), 102)
    ks = O.block_summary(kc)
    o, idx, cnt, lse = O.decode(q, kc, vc, lens, ks, Hkv, topk, gated=gated)
    sidx, scnt, slogg, _ = O.select_decode(q, ks, lens, Hkv, topk)
    assert np.array_equal(idx, sidx) and np.array_equal(cnt, scnt)
    for b in range(B):
        n = lens[b]
        t = (n - 1) // 64
        assert cnt[b, 0] == min(topk, t)
        for h in range(Hq):
            r = h // 2
            mask = torch.full((L,), float("-inf"), dtype=torch.float64)
            for s in range(cnt[b, r]):
                m = idx[b, r, s]
                mask[m * 64:(m + 1) * 64] = slogg[b, r, s] if gated else 0.0
            mask[t * 64:n] = 0.0
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, h])[None, None, None], torch.from_numpy(kc[b, r])[None, None],
                torch.from_numpy(vc[b, r])[None, None], attn_mask=mask[None, None, None])
            assert np.abs(o[b, h] - ref.numpy()[0, 0, 0]).max() < 1e-12


def test_decode_selection_enumeration():
    B, Hq, Hkv, L, d = 1, 4, 1, 512, 8
    q = rnd((B, Hq, d), 110)
    kc = rnd((B, Hkv, L, d), 111)
    ks = O.block_summary(kc)
    idx, cnt, logg, scores = O.select_decode(q, ks, [L], Hkv, 3)
    qbar = q[0].mean(axis=0)
    s = np.array([qbar @ kc[0, 0, m * 64:(m + 1) * 64].mean(axis=0) / np.sqrt(d) for m in range(7)])
    assert idx[0, 0].tolist() == brute.topk_enumerate(s, 3).tolist()
    assert np.allclose(logg[0, 0], s[idx[0, 0]] - np.log(np.exp(s).sum()), atol=1e-13)


def test_stored_output_form_of_D():
    """attn_bwd with the exact output passed as the stored one is unchanged;
    a rounded stored output moves only the row term D (dv does not use D)."""
    q, k, v, do, idx, cnt, logg = _sparse_case(120, N=256, d=16, topk=2)
    o, _ = O.attn_fwd(q, k, v, idx, cnt, logg)
    ref = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    same = O.attn_bwd(q, k, v, do, idx, cnt, logg, o_stored=o)
    for a, b in zip(ref, same):
        assert np.abs(a - b).max() < 1e-13
    rounded = inputs.to_storage(o, "bf16").double().numpy()
    moved = O.attn_bwd(q, k, v, do, idx, cnt, logg, o_stored=rounded)
    assert np.abs(moved[2] - ref[2]).max() < 1e-13          # dv
    assert 0 < np.abs(moved[3] - ref[3]).max() < 0.05        # dlogg shifts a little
    as_fn = O.attn_bwd(q, k, v, do, idx, cnt, logg,
                       o_stored=lambda rows: inputs.to_storage(rows, "bf16").double().numpy())
    for a, b in zip(moved, as_fn):
        assert np.abs(a - b).max() < 1e-13


# ---------------------------------------------------------------- selector backward pins
def _gated_loss(q, k, v, do, idx, cnt, Hkv):
    """L(q, k) = sum(dO * o) with the selection (idx, cnt) held fixed and the
    gate recomputed from q and k through the selector (summaries, scores,
    log g = s - LSE(s) by the oracle's gate), then gated attention."""
    ks = O.block_summary(k)
    B, Hq, N, d = q.shape
    G = Hq // Hkv
    T = -(-N // BLOCK)
    scale = 1.0 / np.sqrt(d)
    logg = np.zeros(idx.shape)
    for b in range(B):
        for r in range(Hkv):
            for t in range(1, T):
                rows = q[b, r * G:(r + 1) * G, t * BLOCK:min(N, (t + 1) * BLOCK)]
                s = scale * (ks[b, r, :t] @ rows.reshape(-1, d).mean(axis=0))
                _, _, logg_all = O.gate_and_topk(s, 1)
                for j in range(int(cnt[b, r, t])):
                    logg[b, r, t, j] = logg_all[idx[b, r, t, j]]
    o, _ = O.attn_fwd(q, k, v, idx, cnt, logg)
    return (o * do).sum(), logg


def test_selector_backward_central_finite_differences():
    """Attention backward + selector backward (eq. 8 through the parameter-free
    selector) = the numerical gradient of the loss with the selection fixed;
    the attention part alone does not match."""
    Hkv = 2
    q, k, v, do, idx, cnt, logg = _sparse_case(80, N=256, d=8, Hq=4, Hkv=Hkv, topk=2)
    _, logg0 = _gated_loss(q, k, v, do, idx, cnt, Hkv)
    assert np.abs(logg0 - logg).max() < 1e-12  # the selection's own gate
    dq_a, dk_a, _, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    dq_s, dk_s = O.select_backward(q, k, idx, cnt, dlogg, Hkv)
    grads = {"q": dq_a + dq_s, "k": dk_a + dk_s}
    alone = {"q": dq_a, "k": dk_a}
    h = 1e-5
    probes = [("q", (0, 1, 150, 3)), ("q", (0, 3, 70, 0)), ("q", (0, 2, 200, 5)),
              ("k", (0, 0, 10, 5)), ("k", (0, 1, 130, 2)), ("k", (0, 1, 70, 7))]
    misses = 0
    for name, ix in probes:
        args = dict(q=q, k=k)
        xp, xm = args[name].copy(), args[name].copy()
        xp[ix] += h
        xm[ix] -= h
        lp, _ = _gated_loss(**{**args, name: xp}, v=v, do=do, idx=idx, cnt=cnt, Hkv=Hkv)
        lm, _ = _gated_loss(**{**args, name: xm}, v=v, do=do, idx=idx, cnt=cnt, Hkv=Hkv)
        fd = (lp - lm) / (2 * h)
        assert abs(fd - grads[name][ix]) <= 1e-7 * max(1.0, abs(fd)), (name, ix, fd, grads[name][ix])
        misses += abs(fd - alone[name][ix]) > 1e-6 * max(1.0, abs(fd))
    assert misses >= 4  # the selector's share is visible at most probes


def test_selector_backward_eq8_structure():
    """Per row: the score gradients sum to zero (softmax normalisation), and
    every block outside the kept set gets -g_m times the kept gradients' sum
    (eq. 8, sparse scope)."""
    Hkv = 2
    q, k, v, do, idx, cnt, logg = _sparse_case(81, N=512, d=16, Hq=4, Hkv=Hkv, topk=3)
    _, _, _, dlogg = O.attn_bwd(q, k, v, do, idx, cnt, logg)
    _, _, ds_rows = O.select_backward(q, k, idx, cnt, dlogg, Hkv, return_ds=True)
    ks = O.block_summary(k)
    assert len(ds_rows) == Hkv * 7
    for (b, r, t), ds in ds_rows.items():
        assert abs(ds.sum()) < 1e-12
        qbar = q[b, r * 2:(r + 1) * 2, t * BLOCK:(t + 1) * BLOCK].reshape(-1, 16).mean(axis=0)
        s = (ks[b, r, :t] @ qbar) / 4.0
        g = np.exp(s - s.max())
        g /= g.sum()
        kk = int(cnt[b, r, t])
        kept = set(int(m) for m in idx[b, r, t, :kk])
        total = dlogg[b, r, t, :kk].sum()
        for m in range(t):
            if m not in kept:
                assert abs(ds[m] + g[m] * total) < 1e-12


# ---------------------------------------------------------------- bf16 summaries
def test_round_bf16_matches_library_conversion():
    """The oracle's bf16 rounding equals torch's float32 -> bfloat16 conversion
    (round to nearest even) on float32 values, including exact midpoints."""
    x = rnd(20000, 97).astype(np.float32) * np.float32(3.0)
    mids = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(2.0 + 2.0 ** -7), 0.5 + 2.0 ** -9,
                     0.0], dtype=np.float32)  # halfway cases tie to the even neighbour
    xs = np.concatenate([x, mids])
    want = torch.from_numpy(xs).to(torch.bfloat16).double().numpy()
    got = O.round_bf16(xs.astype(np.float64))
    assert np.array_equal(got, want)
    assert got[-5] == 1.0 and got[-4] == 1.0 + 2 * 2.0 ** -7 and got[-3] == -2.0


# ------------------------------------------------------------------ per-token selection
def _tok_case(N, d, Hq, Hkv, topk, seed, const_blocks=False):
    B = 1
    q, k, v, do = (rnd((B, Hq, N, d), seed), rnd((B, Hkv, N, d), seed + 1),
                   rnd((B, Hkv, N, d), seed + 2), rnd((B, Hq, N, d), seed + 3))
    if const_blocks:  # every query block's rows repeat its first row, per head
        for t in range(-(-N // BLOCK)):
            q[:, :, t * BLOCK:(t + 1) * BLOCK] = q[:, :, t * BLOCK:t * BLOCK + 1]
    return q, k, v, do


def test_tokens_equal_blocks_when_queries_are_constant_in_each_block():
    """With q constant across each 64-token query block, every token's own
    selection is its block's selection; outputs and gradients match the
    per-block oracle, and the per-block d(log g) is the sum over the block's
    tokens."""
    N, d, Hq, Hkv, topk = 300, 16, 4, 2, 2
    q, k, v, do = _tok_case(N, d, Hq, Hkv, topk, 900, const_blocks=True)
    ks = O.block_summary(k)
    bi, bc, bl, _ = O.select_prefill(q, ks, Hkv, topk)
    ti, tc, tl, _ = O.select_prefill_tokens(q, ks, Hkv, topk)
    for i in range(N):
        t = i // BLOCK
        assert np.array_equal(ti[:, :, i], bi[:, :, t]) and np.array_equal(tc[:, :, i], bc[:, :, t])
        assert np.allclose(tl[:, :, i], bl[:, :, t], rtol=0, atol=1e-12)
    ob, lb = O.attn_fwd(q, k, v, bi, bc, bl)
    ot, lt = O.attn_fwd_tokens(q, k, v, ti, tc, tl)
    assert np.abs(ob - ot).max() < 1e-12 and np.abs(lb - lt).max() < 1e-12
    gb = O.attn_bwd(q, k, v, do, bi, bc, bl)
    gt = O.attn_bwd_tokens(q, k, v, do, ti, tc, tl)
    for a, b_ in zip(gb[:3], gt[:3]):
        assert np.abs(a - b_).max() < 1e-10
    summed = np.zeros_like(gb[3])
    for i in range(N):
        summed[:, :, i // BLOCK] += gt[3][:, :, i]
    assert np.abs(summed - gb[3]).max() < 1e-10


def test_tokens_forward_against_dense_masked_matrix():
    """Brute force: the whole N x N logit matrix per head with the bias and
    mask each row's selection implies, a softmax per row."""
    N, d, Hq, Hkv, topk = 260, 8, 4, 2, 2
    q, k, v, _ = _tok_case(N, d, Hq, Hkv, topk, 910)
    idx, cnt, logg, _ = O.select_prefill_tokens(q, O.block_summary(k), Hkv, topk)
    o, lse = O.attn_fwd_tokens(q, k, v, idx, cnt, logg)
    G = Hq // Hkv
    scale = 1.0 / np.sqrt(d)
    blk = np.arange(N) // BLOCK
    for h in range(Hq):
        r = h // G
        bias = np.full((N, N), -np.inf)
        for i in range(N):
            for slot in range(int(cnt[0, r, i])):
                bias[i, blk == idx[0, r, i, slot]] = logg[0, r, i, slot]
            cur = (blk == i // BLOCK) & (np.arange(N) <= i)
            bias[i, cur] = 0.0
        z = scale * (q[0, h] @ k[0, r].T) + bias
        zmax = z.max(axis=1, keepdims=True)
        p = np.exp(z - zmax)
        assert np.abs(p / p.sum(axis=1, keepdims=True) @ v[0, r] - o[0, h]).max() < 1e-12
        assert np.abs(zmax[:, 0] + np.log(p.sum(axis=1)) - lse[0, h]).max() < 1e-12


def test_tokens_backward_central_finite_differences():
    """dq, dk, dv and d(log g) of L = sum(dO * o) against central differences
    (the selection held fixed; log g perturbed as an input)."""
    N, d, Hq, Hkv, topk = 140, 4, 2, 1, 1
    q, k, v, do = _tok_case(N, d, Hq, Hkv, topk, 920)
    idx, cnt, logg, _ = O.select_prefill_tokens(q, O.block_summary(k), Hkv, topk)
    dq, dk, dv, dlogg = O.attn_bwd_tokens(q, k, v, do, idx, cnt, logg)

    def loss(q_, k_, v_, lg_):
        return float((O.attn_fwd_tokens(q_, k_, v_, idx, cnt, lg_)[0] * do).sum())

    eps = 1e-6
    rng = np.random.Generator(np.random.PCG64(921))
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("logg", logg, dlogg)):
        flat = np.flatnonzero(cnt[..., None].repeat(topk, -1) > 0) if name == "logg" else None
        for _ in range(4):
            if name == "logg":
                e = np.unravel_index(int(rng.choice(flat)), arr.shape)
            else:
                e = tuple(int(rng.integers(0, s)) for s in arr.shape)
            hi, lo = arr.copy(), arr.copy()
            hi[e] += eps
            lo[e] -= eps
            args = {"q": (q, k, v, logg), "k": (q, k, v, logg), "v": (q, k, v, logg),
                    "logg": (q, k, v, logg)}[name]
            pos = list(args)
            slot = ["q", "k", "v", "logg"].index(name)
            pos[slot] = hi
            up = loss(*pos)
            pos[slot] = lo
            dn = loss(*pos)
            num = (up - dn) / (2 * eps)
            assert abs(num - grad[e]) < 1e-6 * max(1.0, abs(num)), (name, e, num, grad[e])


def _tokens_gated_loss(q, k, v, do, idx, cnt, Hkv):
    """L(q, k) = sum(dO * o) with the per-token selection held fixed and each
    token's gate recomputed from q and k (summaries, scores, log g)."""
    ks = O.block_summary(k)
    B, Hq, N, d = q.shape
    G = Hq // Hkv
    logg = np.zeros(idx.shape)
    for b in range(B):
        for r in range(Hkv):
            for i in range(BLOCK, N):
                s = (ks[b, r, :i // BLOCK] @ q[b, r * G:(r + 1) * G, i].mean(axis=0)) / np.sqrt(d)
                _, _, logg_all = O.gate_and_topk(s, 1)
                for j in range(int(cnt[b, r, i])):
                    logg[b, r, i, j] = logg_all[idx[b, r, i, j]]
    o, _ = O.attn_fwd_tokens(q, k, v, idx, cnt, logg)
    return (o * do).sum(), logg


def test_tokens_selector_backward_central_finite_differences():
    """Per-token attention backward + per-token selector backward = the
    numerical gradient of the loss with the selection fixed."""
    N, d, Hq, Hkv, topk = 200, 8, 4, 2, 2
    q, k, v, do = _tok_case(N, d, Hq, Hkv, topk, 930)
    idx, cnt, logg, _ = O.select_prefill_tokens(q, O.block_summary(k), Hkv, topk)
    _, logg0 = _tokens_gated_loss(q, k, v, do, idx, cnt, Hkv)
    assert np.abs(logg0 - logg).max() < 1e-12
    dq_a, dk_a, _, dlogg = O.attn_bwd_tokens(q, k, v, do, idx, cnt, logg)
    dq_s, dk_s = O.select_backward_tokens(q, k, idx, cnt, dlogg, Hkv)
    grads = {"q": dq_a + dq_s, "k": dk_a + dk_s}
    h = 1e-5
    misses = 0
    for name, ix in (("q", (0, 1, 150, 3)), ("q", (0, 3, 70, 0)), ("q", (0, 2, 199, 5)),
                     ("k", (0, 0, 10, 5)), ("k", (0, 1, 100, 2)), ("k", (0, 1, 70, 7))):
        args = dict(q=q, k=k)
        xp, xm = args[name].copy(), args[name].copy()
        xp[ix] += h
        xm[ix] -= h
        lp, _ = _tokens_gated_loss(**{**args, name: xp}, v=v, do=do, idx=idx, cnt=cnt, Hkv=Hkv)
        lm, _ = _tokens_gated_loss(**{**args, name: xm}, v=v, do=do, idx=idx, cnt=cnt, Hkv=Hkv)
        fd = (lp - lm) / (2 * h)
        assert abs(fd - grads[name][ix]) <= 1e-7 * max(1.0, abs(fd)), (name, ix, fd, grads[name][ix])
        misses += abs(fd - (dq_a if name == "q" else dk_a)[ix]) > 1e-6 * max(1.0, abs(fd))
    assert misses >= 3  # the selector's share is visible
