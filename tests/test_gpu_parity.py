"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Bars: block indices and counts bit-exact; floating-point outputs within
max-abs 2e-2 for bf16 data and 1e-4 for fp32 data (o, lse, dq, dk, dv, dlogg,
log g). An output stored in bf16 cannot be nearer the fp64 value than its own
rounding to nearest: bf16 keeps 8 significant bits, so rounding moves x by at
most half an ulp, 2^(floor(log2|x|) - 8) (between 2^-9 |x| and 2^-8 |x|).
For those outputs (o, dq, dk, dv) each element may exceed the absolute bound
by exactly that half ulp (of the larger of |got| and |ref|) and no more.
fp32-stored outputs (lse, dlogg, log g, raw scores) get the plain bound.
Every check records the plain max-abs error of its output; the run prints
them at the end. Summaries are fp32 sums of 64 values: 1e-5.

The backward's row term is D_i = dO_i . o_i with o as the forward stored it
(the interface passes the stored output in). In the small-case checks both
backwards receive the oracle's forward outputs as stored (o rounded to the
storage dtype, lse in fp32); the c3 check runs forward and backward end to
end on the GPU.

Both sides consume the same stored bytes: the seeded generators produce
bf16/fp32 tensors, the oracle upcasts them to fp64. Where a test feeds a
selection to the attention kernels it is the oracle's (idx, cnt, and log g
rounded to fp32), so the attention parity does not depend on the selection
parity, which is tested on its own.
"""
import numpy as np
import pytest
import torch

import parity_report
from gated_block_sparse_b200 import inputs, sas
from oracle import sas_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {"bf16": 2e-2, "f32": 1e-4}


def dev(t):
    return t.to(DEV).contiguous()


def np64(t):
    return t.detach().cpu().double().numpy()


def maxerr(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    return 0.0 if a.size == 0 else float(np.abs(a - b).max())


def half_ulp_bf16(x):
    """Half an ulp of bf16 at |x|: 2^(floor(log2|x|) - 8) (0 at x = 0), the
    most that rounding to nearest bf16 moves a value of that magnitude."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(x > 0, x, 1.0)))
    return np.where(x > 0, np.ldexp(1.0, (e - 8).astype(np.int64)), 0.0)


def excess(got, ref, base, stored_bf16, name=None):
    """Largest |got - ref| beyond the bound (<= 0 passes): base, plus half a
    bf16 ulp (at the larger of |got| and |ref|) for outputs stored in bf16.
    With `name`, the plain max-abs error is recorded for the end-of-run
    report."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return -base
    err = np.abs(got - ref)
    bound = base + half_ulp_bf16(np.maximum(np.abs(got), np.abs(ref))) if stored_bf16 else base
    ex = float((err - bound).max())
    if name is not None:
        import os
        test = os.environ.get("PYTEST_CURRENT_TEST", "?").split("::")[-1].split(" ")[0]
        parity_report.record(test, name, float(err.max()),
                             f"{base:g}" + (" + half ulp" if stored_bf16 else ""), ex,
                             float(np.abs(ref).max()))
    return ex


def stored(dtype):
    return lambda rows: inputs.to_storage(rows, dtype).double().numpy()


def boundary_gap(scores: dict, topk: int) -> float:
    g = np.inf
    for s in scores.values():
        if len(s) > topk:
            ss = np.sort(s)[::-1]
            g = min(g, ss[topk - 1] - ss[topk])
    return g


def oracle_selection(q, k, Hkv, topk):
    ks = O.block_summary(k)
    idx, cnt, logg, scores = O.select_prefill(q, ks, Hkv, topk)
    return idx, cnt, logg.astype(np.float32), scores


# ------------------------------------------------------------------ summaries
@pytest.mark.parametrize("dtype,d,N", [("bf16", 128, 1000), ("f32", 64, 640), ("bf16", 64, 64),
                                       ("f32", 128, 130)])
def test_block_summary(dtype, d, N):
    k = inputs.gen_prefill(2, 2, 2, N, d, dtype, seed=11)["k"]
    got = sas.sas_block_summary(dev(k))
    torch.cuda.synchronize()
    assert maxerr(np64(got), O.block_summary(k)) < 1e-5


def test_block_summary_lens():
    k = inputs.gen_prefill(3, 2, 2, 512, 128, "bf16", seed=12)["k"]
    lens = torch.tensor([512, 200, 1], dtype=torch.int32)
    got = sas.sas_block_summary(dev(k), lens=dev(lens))
    torch.cuda.synchronize()
    assert maxerr(np64(got), O.block_summary(k, lens=lens.numpy())) < 1e-5



def _bf16_ulp(x):
    e = np.frexp(np.where(x == 0, 1.0, x))[1]
    return np.ldexp(1.0, e - 8)


@pytest.mark.parametrize("dtype,d,N", [("bf16", 128, 1000), ("f32", 64, 640)])
def test_block_summary_bf16(dtype, d, N):
    """Summaries stored in bf16: the kernel's fp32 mean (within 1e-5 of the
    exact one) rounded to nearest even, against the exact mean rounded. They
    may differ only where the exact mean lies that close to a halfway point,
    and then by one bf16 ulp."""
    k = inputs.gen_prefill(2, 2, 2, N, d, dtype, seed=13)["k"]
    got = sas.sas_block_summary_ex(dev(k), torch.bfloat16)
    torch.cuda.synchronize()
    assert got.dtype == torch.bfloat16
    ref = O.round_bf16(O.block_summary(k))
    diff = np.abs(np64(got) - ref)
    assert np.all(diff <= _bf16_ulp(ref) * 1.0001)
    assert (diff > 0).mean() < 1e-3
    f32 = sas.sas_block_summary_ex(dev(k), torch.float32)
    assert torch.equal(f32, sas.sas_block_summary(dev(k)))

# ------------------------------------------------------------------ selection
def dense_scores(scores: dict, shape) -> np.ndarray:
    """The oracle's per-row score arrays laid out as the library's raw-score
    output: row key (b, r[, t]) -> its C scores, -inf past C."""
    out = np.full(shape, -np.inf)
    for key, s in scores.items():
        out[key][:len(s)] = s
    return out


def _check_scores(got, scores: dict, tol=1e-5):
    ref = dense_scores(scores, tuple(got.shape))
    g = np64(got)
    assert np.array_equal(np.isinf(g), np.isinf(ref)) and np.all(g[np.isinf(g)] < 0)
    fin = np.isfinite(ref)
    assert excess(g[fin], ref[fin], tol, False, "scores") <= 0


def _check_select(q, k, Hkv, topk, tol):
    ks = sas.sas_block_summary(dev(k))
    B, N = q.shape[0], q.shape[2]
    T = -(-N // 64)
    sc = torch.empty((B, Hkv, T, T), dtype=torch.float32, device=DEV)
    idx, cnt, logg = sas.sas_select(dev(q), ks, Hkv, topk, "prefill", scores_out=sc)
    torch.cuda.synchronize()
    oi, oc, ol, scores = oracle_selection(q, k, Hkv, topk)
    assert np.array_equal(cnt.cpu().numpy(), oc)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert excess(np64(logg), ol, tol, False, "logg") <= 0
    _check_scores(sc, scores)
    return scores


def test_select_prefill_c1():
    x = inputs.gen_config("c1")
    c = inputs.CONFIGS["c1"]
    scores = _check_select(x["q"], x["k"], c["Hkv"], c["topk"], 1e-5)
    assert boundary_gap(scores, c["topk"]) >= 1.5e-3


@pytest.mark.parametrize("N,d,topk", [(2048, 128, 7), (1000, 64, 3), (4096, 128, 31)])
def test_select_prefill_planted_bf16(N, d, topk):
    x = inputs.gen_prefill(2, 8, 2, N, d, "bf16", seed=20 + N, plant="ramp")
    scores = _check_select(x["q"], x["k"], 2, topk, 1e-4)
    assert boundary_gap(scores, topk) >= 1.5e-3


def test_select_prefill_many_chunks():
    # C up to 319 history blocks: two score chunks and a list merge per row
    x = inputs.gen_prefill(1, 2, 1, 20480, 64, "bf16", seed=33, plant="ramp")
    scores = _check_select(x["q"], x["k"], 1, 40, 1e-4)
    assert boundary_gap(scores, 40) >= 1.5e-3


def test_select_prefill_exact_ties():
    x = inputs.gen_prefill(1, 4, 2, 1024, 128, "bf16", seed=34)
    k = torch.zeros_like(x["k"])
    _check_select(x["q"], k, 2, 5, 1e-5)  # all scores 0: lowest indices, log g = -log C


def test_select_prefill_topk_zero():
    x = inputs.gen_prefill(1, 4, 2, 512, 64, "f32", seed=35)
    ks = sas.sas_block_summary(dev(x["k"]))
    idx, cnt, logg = sas.sas_select(dev(x["q"]), ks, 2, 0, "prefill")
    torch.cuda.synchronize()
    assert int(cnt.abs().sum()) == 0


# ------------------------------------------------------------------ attention
def _fwd_bwd_check(x, Hkv, topk, dtype, sel=None):
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    if sel is None:
        sel = oracle_selection(q, k, Hkv, topk)
    idx, cnt, logg = sel[:3]
    dq_, dk_, dv_, do_ = dev(q), dev(k), dev(v), dev(do)
    ti, tc, tl = dev(torch.from_numpy(idx)), dev(torch.from_numpy(cnt)), dev(torch.from_numpy(logg))
    o, lse = sas.sas_attn_fwd(dq_, dk_, dv_, ti, tc, tl)
    oo, olse = O.attn_fwd(q, k, v, idx, cnt, logg)
    # The backward is checked on the forward outputs as stored by the oracle
    # (o rounded to the storage dtype, lse in fp32), so that its check does not
    # depend on how the GPU forward rounded; the forward is checked above it.
    o_in = dev(inputs.to_storage(oo, dtype))
    lse_in = dev(torch.from_numpy(olse.astype(np.float32)))
    gq, gk, gv, gl = sas.sas_attn_bwd(dq_, dk_, dv_, o_in, do_, lse_in, ti, tc, tl)
    torch.cuda.synchronize()
    oq, okk, ov, ol = O.attn_bwd(q, k, v, do, idx, cnt, logg, o_stored=stored(dtype))
    tol = TOL[dtype]
    bf = dtype == "bf16"
    errs = dict(o=excess(np64(o), oo, tol, bf, "o"), lse=excess(np64(lse), olse, tol, False, "lse"),
                dq=excess(np64(gq), oq, tol, bf, "dq"), dk=excess(np64(gk), okk, tol, bf, "dk"),
                dv=excess(np64(gv), ov, tol, bf, "dv"),
                dlogg=excess(np64(gl), ol, tol, False, "dlogg"))
    for name, e in errs.items():
        assert e <= 0, (name, e, errs)
    return errs


def test_attn_c1_fp32():
    c = inputs.CONFIGS["c1"]
    _fwd_bwd_check(inputs.gen_config("c1"), c["Hkv"], c["topk"], "f32")


@pytest.mark.parametrize("B,Hq,Hkv,N,d,topk", [(1, 8, 2, 1000, 128, 3), (2, 4, 4, 576, 64, 2),
                                               (1, 8, 1, 768, 128, 5)])
def test_attn_bf16_ragged(B, Hq, Hkv, N, d, topk):
    x = inputs.gen_prefill(B, Hq, Hkv, N, d, "bf16", seed=40 + N)
    _fwd_bwd_check(x, Hkv, topk, "bf16")


def test_attn_dense_equivalence_bf16():
    # every history block selected and log g = 0: plain causal attention
    x = inputs.gen_prefill(1, 4, 2, 512, 128, "bf16", seed=50)
    T = 8
    idx = np.full((1, 2, T, T), -1, dtype=np.int32)
    cnt = np.zeros((1, 2, T), dtype=np.int32)
    for t in range(T):
        idx[:, :, t, :t] = np.arange(t)
        cnt[:, :, t] = t
    _fwd_bwd_check(x, 2, T, "bf16", sel=(idx, cnt, np.zeros((1, 2, T, T), np.float32)))


def test_attn_topk_zero_current_block_only():
    x = inputs.gen_prefill(1, 2, 2, 256, 64, "f32", seed=51)
    sel = (np.zeros((1, 2, 4, 0), np.int32), np.zeros((1, 2, 4), np.int32),
           np.zeros((1, 2, 4, 0), np.float32))
    q, k, v = (dev(x[n]) for n in ("q", "k", "v"))
    o, lse = sas.sas_attn_fwd(q, k, v, dev(torch.zeros(1, 2, 4, 1, dtype=torch.int32))[..., :0],
                              dev(torch.from_numpy(sel[1])),
                              dev(torch.zeros(1, 2, 4, 1))[..., :0])
    torch.cuda.synchronize()
    oo, olse = O.attn_fwd(x["q"], x["k"], x["v"], *sel)
    assert maxerr(np64(o), oo) < 1e-4 and maxerr(np64(lse), olse) < 1e-4


def test_attn_c3_dense():
    """Full c3 workload (N = 16384, GQA 32/8, d = 128, top-k 31) in the
    launch configuration the bench times, checked everywhere: selection and
    raw scores on every row; o and lse of every query row and head; then the
    backward, given the forward outputs as the oracle stores them (o rounded
    to bf16, lse in fp32), as in the small cases: dq of every row, dlogg of
    every (kv group, query block) slot, dk and dv of every key. The oracle
    runs all 2048 (kv group, query block) units in a process pool."""
    import oracle_pool
    c = inputs.CONFIGS["c3"]
    x = inputs.gen_config("c3")
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    ks = sas.sas_block_summary(dev(k))
    T = 256
    sc = torch.empty((1, c["Hkv"], T, T), dtype=torch.float32, device=DEV)
    ti, tc, tl = sas.sas_select(dev(q), ks, c["Hkv"], c["topk"], "prefill", scores_out=sc)
    o, lse = sas.sas_attn_fwd(dev(q), dev(k), dev(v), ti, tc, tl)
    torch.cuda.synchronize()
    oi, oc, ol, scores = oracle_selection(q, k, c["Hkv"], c["topk"])
    assert boundary_gap(scores, c["topk"]) >= 1.5e-3
    assert np.array_equal(tc.cpu().numpy(), oc) and np.array_equal(ti.cpu().numpy(), oi)
    assert excess(np64(tl), ol, 1e-4, False, "logg") <= 0
    _check_scores(sc, scores)
    ref = oracle_pool.prefill_all(q, k, v, do, oi, oc, ol.astype(np.float32), "bf16")
    tol = TOL["bf16"]
    assert excess(np64(o), ref["o"], tol, True, "o") <= 0
    assert excess(np64(lse), ref["lse"], tol, False, "lse") <= 0
    o_in = dev(inputs.to_storage(ref["o"], "bf16"))
    lse_in = dev(torch.from_numpy(ref["lse"].astype(np.float32)))
    gq, gk, gv, gl = sas.sas_attn_bwd(dev(q), dev(k), dev(v), o_in, dev(do), lse_in, ti, tc, tl)
    torch.cuda.synchronize()
    st, msg = sas.sas_device_status()
    assert st == 0, msg
    for name, got, bf in (("dq", gq, True), ("dk", gk, True), ("dv", gv, True),
                          ("dlogg", gl, False)):
        e = excess(np64(got), ref[name], tol, bf, name)
        assert e <= 0, (name, e)


# ------------------------------------------------------------------ decode
def _decode_check(x, Hkv, topk, gated, tol=2e-2):
    q, kc, vc, lens = x["q"], x["kc"], x["vc"], x["lens"]
    ks = sas.sas_block_summary(dev(kc))
    idx_out = torch.empty((q.shape[0], Hkv, topk), dtype=torch.int32, device=DEV)
    o = sas.sas_decode(dev(q), dev(kc), dev(vc), dev(lens), ks, topk, gated=gated,
                       idx_out=idx_out if topk else None)
    torch.cuda.synchronize()
    oks = O.block_summary(kc)
    assert maxerr(np64(ks), oks) < 1e-5
    oo, oi, oc, _ = O.decode(q, kc, vc, lens.numpy(), oks, Hkv, topk, gated=gated)
    if topk:
        assert np.array_equal(idx_out.cpu().numpy(), oi)
    err = excess(np64(o), oo, tol, q.dtype == torch.bfloat16, "o")
    assert err <= 0, err
    _, _, _, scores = O.select_decode(q, oks, lens.numpy(), Hkv, topk)
    return scores


@pytest.mark.parametrize("case", ["c2", "ragged"])
def test_select_decode_rows_and_scores(case):
    """sas_select in decode mode (the split path's selection): indices, counts
    and log g of every row, and the raw scores against the oracle's."""
    if case == "c2":
        c = inputs.CONFIGS["c2"]
        x, Hkv, topk = inputs.gen_config("c2"), c["Hkv"], c["topk"]
    else:
        x, Hkv, topk = inputs.gen_decode(4, 8, 2, 1024, 128, [1, 64, 65, 1024], "bf16", seed=60,
                                         planted=8), 2, 4
    q, kc, lens = x["q"], x["kc"], x["lens"]
    ks = sas.sas_block_summary(dev(kc))
    B, nblk = q.shape[0], kc.shape[2] // 64
    sc = torch.empty((B, Hkv, nblk), dtype=torch.float32, device=DEV)
    idx, cnt, logg = sas.sas_select(dev(q), ks, Hkv, topk, "decode", lens=dev(lens),
                                    scores_out=sc)
    torch.cuda.synchronize()
    oi, oc, ol, scores = O.select_decode(q, O.block_summary(kc), lens.numpy(), Hkv, topk)
    assert np.array_equal(cnt.cpu().numpy(), oc) and np.array_equal(idx.cpu().numpy(), oi)
    assert excess(np64(logg), ol, 1e-4, False, "logg") <= 0
    _check_scores(sc, scores)


@pytest.mark.parametrize("gated", [1, 0])
def test_decode_c2(gated):
    c = inputs.CONFIGS["c2"]
    scores = _decode_check(inputs.gen_config("c2"), c["Hkv"], c["topk"], gated)
    assert boundary_gap(scores, c["topk"]) >= 1.5e-3


@pytest.mark.parametrize("lens", [[1, 64, 65, 1024], [700, 128, 1000, 63]])
def test_decode_ragged_small(lens):
    x = inputs.gen_decode(4, 8, 2, 1024, 128, lens, "bf16", seed=60, planted=8)
    scores = _decode_check(x, 2, 4, 1)
    assert boundary_gap(scores, 4) >= 1.5e-3


@pytest.mark.parametrize("G,d,dtype", [(1, 64, "f32"), (2, 128, "f32"), (8, 64, "bf16")])
def test_decode_group_sizes(G, d, dtype):
    x = inputs.gen_decode(2, 2 * G, 2, 2048, d, [2048, 1500], dtype, seed=61, planted=6)
    _decode_check(x, 2, 5, 1, tol=TOL[dtype])


def test_decode_exact_ties():
    x = inputs.gen_decode(1, 32, 8, 4096, 128, [4000], "bf16", seed=62)
    x["kc"] = torch.zeros_like(x["kc"])
    _decode_check(x, 8, 15, 1)


def test_decode_topk_zero():
    x = inputs.gen_decode(2, 8, 2, 512, 64, [300, 512], "bf16", seed=63)
    _decode_check(x, 2, 0, 1)


@pytest.mark.parametrize("name", ["c4", "c5"])
def test_decode_full_configs(name):
    c = inputs.CONFIGS[name]
    scores = _decode_check(inputs.gen_config(name), c["Hkv"], c["topk"], c["gated"])
    assert boundary_gap(scores, c["topk"]) >= 1.5e-3



def _decode_bf16_summary_check(x, Hkv, topk, gated, tol=2e-2):
    q, kc, vc, lens = x["q"], x["kc"], x["vc"], x["lens"]
    ks = sas.sas_block_summary_ex(dev(kc), torch.bfloat16, lens=dev(lens))
    idx = torch.empty((q.shape[0], Hkv, topk), dtype=torch.int32, device=DEV)
    o = sas.sas_decode_ex(dev(q), dev(kc), dev(vc), dev(lens), ks, topk, gated=gated,
                          idx_out=idx if topk else None)
    torch.cuda.synchronize()
    oks = O.round_bf16(O.block_summary(kc, lens=lens.numpy()))
    oo, oi, _, _ = O.decode(q, kc, vc, lens.numpy(), oks, Hkv, topk, gated=gated)
    if topk:
        assert np.array_equal(idx.cpu().numpy(), oi)
    err = excess(np64(o), oo, tol, q.dtype == torch.bfloat16, "o")
    assert err <= 0, err
    _, _, _, scores = O.select_decode(q, oks, lens.numpy(), Hkv, topk)
    return scores


@pytest.mark.parametrize("name", ["c2", "c5"])
def test_decode_bf16_summaries_full_configs(name):
    """Decode reading bf16 summaries against the oracle scoring the exact
    means rounded to bf16 (selection on the stored summaries)."""
    c = inputs.CONFIGS[name]
    scores = _decode_bf16_summary_check(inputs.gen_config(name), c["Hkv"], c["topk"], c["gated"])
    assert boundary_gap(scores, c["topk"]) >= 1.5e-3


@pytest.mark.parametrize("G,d,dtype,lens", [(1, 64, "f32", [2048, 1500]),
                                            (4, 128, "bf16", [700, 65]),
                                            (8, 64, "bf16", [1, 2048])])
def test_decode_bf16_summaries_small(G, d, dtype, lens):
    x = inputs.gen_decode(2, 2 * G, 2, 2048, d, lens, dtype, seed=64, planted=6)
    _decode_bf16_summary_check(x, 2, 5, 1, tol=TOL[dtype])

@pytest.mark.parametrize("Lmax,d,topk,G", [(589824, 64, 63, 2), (262144, 128, 128, 4)])
def test_decode_long_rows_and_large_topk(Lmax, d, topk, G):
    """One long row: more than 512 history blocks per CTA of the cluster (the
    per-CTA list then comes from a sampled bound), and the largest top-k (128:
    lists longer than one warp's sorted share)."""
    x = inputs.gen_decode(1, G, 1, Lmax, d, [Lmax - 5], "bf16", seed=66, planted=2 * topk)
    scores = _decode_check(x, 1, topk, 1)
    assert boundary_gap(scores, topk) >= 1.5e-3

def test_decode_repeat_is_bitwise_stable():
    x = inputs.gen_decode(1, 32, 8, 8192, 128, [8100], "bf16", seed=64, planted=16)
    ks = sas.sas_block_summary(dev(x["kc"]))
    args = (dev(x["q"]), dev(x["kc"]), dev(x["vc"]), dev(x["lens"]), ks, 15)
    a = sas.sas_decode(*args).clone()
    b = sas.sas_decode(*args)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_decode_attend_forced_selection():
    """Decode attention with an arbitrary selection and arbitrary gates."""
    B, Hq, Hkv, L, d, topk = 2, 8, 2, 2048, 128, 6
    x = inputs.gen_decode(B, Hq, Hkv, L, d, [2048, 1111], "bf16", seed=66)
    rng = np.random.Generator(np.random.PCG64(67))
    idx = np.full((B, Hkv, topk), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    logg = np.zeros((B, Hkv, topk), np.float32)
    for b, n in enumerate([2048, 1111]):
        C = (n - 1) // 64
        for r in range(Hkv):
            kk = int(rng.integers(0, topk + 1))
            idx[b, r, :kk] = np.sort(rng.choice(C, kk, replace=False))
            cnt[b, r] = kk
            logg[b, r, :kk] = rng.uniform(-6, 0, kk)
    for gated in (1, 0):
        o = sas.sas_decode_attend(dev(x["q"]), dev(x["kc"]), dev(x["vc"]), dev(x["lens"]),
                                  dev(torch.from_numpy(idx)), dev(torch.from_numpy(cnt)),
                                  dev(torch.from_numpy(logg)), gated=gated)
        torch.cuda.synchronize()
        ref, _ = O.decode_attend(x["q"], x["kc"], x["vc"], x["lens"].numpy(), idx, cnt, logg,
                                 Hkv, gated=gated)
        assert excess(np64(o), ref, 2e-2, True) <= 0


# ---------------------------------------------------------------- selector backward
def _select_bwd_case(B, Hq, Hkv, N, d, dtype, topk, seed):
    x = inputs.gen_prefill(B, Hq, Hkv, N, d, dtype, seed=seed)
    q, k = x["q"], x["k"]
    ks_ref = O.block_summary(k)
    idx, cnt, _, _ = O.select_prefill(q, ks_ref, Hkv, topk)
    T = -(-N // 64)
    rng = np.random.Generator(np.random.PCG64(seed + 7))
    dlogg = rng.standard_normal((B, Hkv, T, topk)).astype(np.float32)
    for b in range(B):  # slots past cnt carry no gradient
        for r in range(Hkv):
            for t in range(T):
                dlogg[b, r, t, cnt[b, r, t]:] = 0.0
    dq_ref, dk_ref = O.select_backward(q, k, idx, cnt, dlogg, Hkv)
    return q, k, idx, cnt, dlogg, dq_ref, dk_ref


@pytest.mark.parametrize("N,d", [(512, 64), (1000, 128)])
def test_select_bwd_fp32(N, d):
    """Eq. 8 through the selector, fp32: relative error at fp32 accumulation level."""
    q, k, idx, cnt, dlogg, dq_ref, dk_ref = _select_bwd_case(2, 8, 2, N, d, "f32", 3, 90 + N)
    qd, kd = q.to(DEV), k.to(DEV)
    ks = sas.sas_block_summary(kd)
    dq = torch.zeros_like(qd)
    dk = torch.zeros_like(kd)
    sas.sas_select_bwd(qd, ks, 2, torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV),
                       torch.from_numpy(dlogg).to(DEV), dq, dk)
    torch.cuda.synchronize()
    for got, ref in ((dq, dq_ref), (dk, dk_ref)):
        g = got.double().cpu().numpy()
        scale_ = np.abs(ref).max()
        assert scale_ > 0
        assert np.abs(g - ref).max() <= 1e-5 * scale_ + 1e-7, np.abs(g - ref).max() / scale_


def test_select_bwd_bf16_adds_in_place():
    """bf16 ragged case; dq and dk start from nonzero values and receive the
    selector's gradient added in place (one bf16 rounding of the sum)."""
    B, Hq, Hkv, N, d = 1, 8, 2, 1000, 128
    q, k, idx, cnt, dlogg, dq_ref, dk_ref = _select_bwd_case(B, Hq, Hkv, N, d, "bf16", 3, 95)
    qd, kd = q.to(DEV), k.to(DEV)
    ks = sas.sas_block_summary(kd)
    g0 = torch.Generator().manual_seed(5)
    dq0 = (torch.randn(q.shape, generator=g0) * 1e-2).to(torch.bfloat16)
    dk0 = (torch.randn(k.shape, generator=g0) * 1e-2).to(torch.bfloat16)
    dq, dk = dq0.to(DEV), dk0.to(DEV)
    sas.sas_select_bwd(qd, ks, Hkv, torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV),
                       torch.from_numpy(dlogg).to(DEV), dq, dk)
    torch.cuda.synchronize()
    for got, init, ref in ((dq, dq0, dq_ref), (dk, dk0, dk_ref)):
        want = init.double().numpy() + ref
        g = got.double().cpu().numpy()
        assert np.abs(g - want).max() <= 2.0 ** -8 * np.abs(want).max() + 1e-6


def test_select_bwd_c3_full():
    """Selector backward on the full c3 workload, on the GPU's selection, with
    a seeded random dlogg standing in for the attention backward's (both
    sides read only the slots below cnt): every element of the selector's
    share of dq and dk against the oracle."""
    c = inputs.CONFIGS["c3"]
    x = inputs.gen_config("c3")
    q, k = x["q"], x["k"]
    qd, kd = dev(q), dev(k)
    ks = sas.sas_block_summary(kd)
    ti, tc, tl = sas.sas_select(qd, ks, c["Hkv"], c["topk"], "prefill")
    T = tl.shape[2]
    g = torch.Generator().manual_seed(11)
    dlogg = torch.randn(tl.shape, generator=g)  # both sides use only slots below cnt
    dq = torch.zeros_like(qd)
    dk = torch.zeros_like(kd)
    sas.sas_select_bwd(qd, ks, c["Hkv"], ti, tc, dlogg.to(DEV), dq, dk)
    torch.cuda.synchronize()
    dq_ref, dk_ref = O.select_backward(q, k, ti.cpu().numpy(), tc.cpu().numpy(),
                                       dlogg.numpy(), c["Hkv"])
    assert T == 256
    for got, ref in ((dq, dq_ref), (dk, dk_ref)):
        gg = got.double().cpu().numpy()
        assert np.abs(gg - ref).max() <= 2.0 ** -8 * np.abs(ref).max() + 1e-6


# ---------------------------------------------------------------- paged decode
def _to_pages(kc, vc, lens, seed, share_prefix=None):
    """Scatter contiguous caches [B][Hkv][Lmax][d] into page pools
    [npages][Hkv][64][d] under a random page order; share_prefix=(a, b, n)
    makes sequence b's first n blocks use sequence a's pages."""
    B, Hkv, Lmax, d = kc.shape
    nblk = Lmax // 64
    rng = np.random.Generator(np.random.PCG64(seed))
    npages = B * nblk + 5  # a few pages no sequence uses
    perm = rng.permutation(npages)
    bt = np.zeros((B, nblk), dtype=np.int32)
    kpool = torch.zeros((npages, Hkv, 64, d), dtype=kc.dtype)
    vpool = torch.zeros_like(kpool)
    nxt = 0
    for b in range(B):
        for m in range(nblk):
            if share_prefix and b == share_prefix[1] and m < share_prefix[2]:
                bt[b, m] = bt[share_prefix[0], m]
                continue
            p = int(perm[nxt])
            nxt += 1
            bt[b, m] = p
            kpool[p] = kc[b, :, m * 64:(m + 1) * 64]
            vpool[p] = vc[b, :, m * 64:(m + 1) * 64]
    return kpool, vpool, bt


@pytest.mark.parametrize("gated", [1, 0])
def test_decode_paged_matches_contiguous_and_oracle(gated):
    """Paged decode against the contiguous kernel (same arithmetic: identical
    selection and output) and against the oracle on the gathered cache; one
    sequence shares a 20-block prefix with another."""
    B, Hq, Hkv, Lmax, d, topk = 3, 32, 8, 8192, 128, 15
    x = inputs.gen_decode(B, Hq, Hkv, Lmax, d, [8192, 5000, 7777], "bf16", seed=71, planted=16)
    q, kc, vc, lens = x["q"], x["kc"].clone(), x["vc"].clone(), x["lens"]
    kc[2, :, :20 * 64] = kc[0, :, :20 * 64]  # the shared prefix has the same content
    vc[2, :, :20 * 64] = vc[0, :, :20 * 64]
    kpool, vpool, bt = _to_pages(kc, vc, lens, seed=72, share_prefix=(0, 2, 20))
    kspool = sas.sas_block_summary(dev(kpool.view(-1, Hkv, 64, d))).view(-1, Hkv, d)
    idx_p = torch.empty((B, Hkv, topk), dtype=torch.int32, device=DEV)
    o_p = sas.sas_decode_paged(dev(q), dev(kpool), dev(vpool), kspool, dev(torch.from_numpy(bt)),
                               dev(lens), topk, gated=gated, idx_out=idx_p)
    ks = sas.sas_block_summary(dev(kc))
    idx_c = torch.empty_like(idx_p)
    o_c = sas.sas_decode(dev(q), dev(kc), dev(vc), dev(lens), ks, topk, gated=gated,
                         idx_out=idx_c)
    torch.cuda.synchronize()
    assert torch.equal(idx_p, idx_c)
    assert torch.equal(o_p, o_c)
    oks = O.block_summary(kc)
    oo, oi, _, _ = O.decode(q, kc, vc, lens.numpy(), oks, Hkv, topk, gated=gated)
    assert np.array_equal(idx_p.cpu().numpy(), oi)
    assert excess(np64(o_p), oo, 2e-2, True) <= 0
    st, msg = sas.sas_device_status()
    assert st == 0, msg


@pytest.mark.parametrize("sum_dtype", [torch.bfloat16, torch.float32])
def test_decode_paged_ex_summary_dtypes(sum_dtype):
    """Paged decode reading page summaries of either dtype: identical to the
    contiguous call reading the same summaries (sas_decode_ex), and against the
    oracle selecting on the stored (for bf16: rounded) means."""
    B, Hq, Hkv, Lmax, d, topk = 2, 16, 4, 8192, 128, 15
    x = inputs.gen_decode(B, Hq, Hkv, Lmax, d, [8192, 6001], "bf16", seed=74, planted=16)
    q, kc, vc, lens = x["q"], x["kc"], x["vc"], x["lens"]
    kpool, vpool, bt = _to_pages(kc, vc, lens, seed=75)
    kspool = sas.sas_block_summary_ex(dev(kpool.view(-1, Hkv, 64, d)), sum_dtype).view(-1, Hkv, d)
    idx_p = torch.empty((B, Hkv, topk), dtype=torch.int32, device=DEV)
    o_p = sas.sas_decode_paged_ex(dev(q), dev(kpool), dev(vpool), kspool,
                                  dev(torch.from_numpy(bt)), dev(lens), topk, idx_out=idx_p)
    ks = sas.sas_block_summary_ex(dev(kc), sum_dtype)
    idx_c = torch.empty_like(idx_p)
    o_c = sas.sas_decode_ex(dev(q), dev(kc), dev(vc), dev(lens), ks, topk, idx_out=idx_c)
    torch.cuda.synchronize()
    assert torch.equal(idx_p, idx_c)
    assert torch.equal(o_p, o_c)
    oks = O.block_summary(kc)
    if sum_dtype == torch.bfloat16:
        oks = O.round_bf16(oks)
    oo, oi, _, _ = O.decode(q, kc, vc, lens.numpy(), oks, Hkv, topk, gated=1)
    assert np.array_equal(idx_p.cpu().numpy(), oi)
    assert excess(np64(o_p), oo, 2e-2, True) <= 0
    st, msg = sas.sas_device_status()
    assert st == 0, msg


def test_decode_host_buffers_match_device_call():
    """sas_decode_host gives the device call's output exactly, with pinned
    host q and o (read and written by the step over the bus) and with
    pageable ones (copied through the device staging buffers)."""
    x = inputs.gen_decode(2, 32, 8, 4096, 128, [4096, 3000], "bf16", seed=73, planted=8)
    q, kc, vc, lens = x["q"], dev(x["kc"]), dev(x["vc"]), dev(x["lens"])
    ks = sas.sas_block_summary(kc)
    o_ref = sas.sas_decode(dev(q), kc, vc, lens, ks, 15).cpu()
    qh = q.clone().pin_memory()
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    qd = torch.empty(q.shape, dtype=q.dtype, device=DEV)
    od = torch.empty_like(qd)
    sas.sas_decode_host(qh, qd, kc, vc, lens, ks, 15, od, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh, o_ref)
    # pageable host buffers: q is copied in through q_dev, o copied out of o_dev
    qp = q.clone()
    op = torch.empty(q.shape, dtype=q.dtype)
    qd.zero_()
    sas.sas_decode_host(qp, qd, kc, vc, lens, ks, 15, od, op)
    torch.cuda.synchronize()
    assert torch.equal(op, o_ref) and torch.equal(qd.cpu(), q)


# ------------------------------------------------------------------ summary upkeep
def _last_block_expect(got, ref, sum_dtype):
    """got, ref: one block's summaries (fp64); bf16 storage allows the one-ulp
    rounding difference of test_block_summary_bf16."""
    if sum_dtype == torch.bfloat16:
        r = O.round_bf16(ref)
        return bool(np.all(np.abs(got - r) <= _bf16_ulp(r) * 1.0001))
    return maxerr(got, ref) < 1e-5


@pytest.mark.parametrize("sum_dtype", [torch.float32, torch.bfloat16])
def test_summary_last_contiguous(sum_dtype):
    """Only each row's last complete block (C - 1, C = (n - 1) // 64) is
    rewritten; rows with C = 0 and every other block keep their contents."""
    B, H, N, d = 4, 2, 1024, 128
    k = inputs.gen_prefill(B, H, H, N, d, "bf16", seed=14)["k"]
    lens = torch.tensor([1, 65, 129, 1000], dtype=torch.int32)  # C = 0, 1, 2, 15
    ks = torch.full((B, H, N // 64, d), 7.0, dtype=sum_dtype, device=DEV)
    sas.sas_block_summary_last(dev(k), dev(lens), ks)
    torch.cuda.synchronize()
    ref, got = O.block_summary(k), np64(ks)
    for b, n in enumerate(lens.tolist()):
        C = (n - 1) // 64
        for m in range(N // 64):
            if m == C - 1:
                assert _last_block_expect(got[b, :, m], ref[b, :, m], sum_dtype)
            else:
                assert (got[b, :, m] == 7.0).all()
    st, msg = sas.sas_device_status()
    assert st == 0, msg


def test_summary_last_paged_and_bad_entry():
    """Paged: the page of block C - 1 gets the summary; a block-table entry
    out of range skips its row and is reported, then cleared."""
    B, H, N, d = 3, 2, 1024, 128
    x = inputs.gen_decode(B, 2 * H, H, N, d, [700, 1024, 64], "bf16", seed=74)
    kc, vc, lens = x["kc"], x["vc"], x["lens"]
    kpool, _, bt = _to_pages(kc, vc, lens, seed=75)
    ks = torch.full((kpool.shape[0], H, d), 7.0, dtype=torch.float32, device=DEV)
    sas.sas_block_summary_last(dev(kpool), dev(lens), ks, block_table=dev(torch.from_numpy(bt)))
    torch.cuda.synchronize()
    ref, got = O.block_summary(kc), np64(ks)
    touched = set()
    for b, n in enumerate(lens.tolist()):
        C = (n - 1) // 64
        if C > 0:
            p = int(bt[b, C - 1])
            touched.add(p)
            assert maxerr(got[p], ref[b, :, C - 1]) < 1e-5
    for p in range(kpool.shape[0]):
        if p not in touched:
            assert (got[p] == 7.0).all()
    st, msg = sas.sas_device_status()
    assert st == 0, msg
    bad = bt.copy()
    bad[1, (1024 - 1) // 64 - 1] = kpool.shape[0]  # one past the pool
    ks2 = torch.full_like(ks, 7.0)
    sas.sas_block_summary_last(dev(kpool), dev(lens), ks2, block_table=dev(torch.from_numpy(bad)))
    st, msg = sas.sas_device_status(clear=True)
    assert st != 0 and "k_summary_last" in msg
    got2 = np64(ks2)
    assert maxerr(got2[int(bt[0, (700 - 1) // 64 - 1])], ref[0, :, (700 - 1) // 64 - 1]) < 1e-5
    assert (got2[int(bt[1, (1024 - 1) // 64 - 1])] == 7.0).all()
    st, msg = sas.sas_device_status()
    assert st == 0, msg
