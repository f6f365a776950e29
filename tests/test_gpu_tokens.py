"""Per-token selection prefill on the GPU against the oracle (CUDA-core path).

Inputs plant block-relevance ramps (gen_prefill, plant='ramp', query shift 4)
so that every token's Top-K boundary gap is at least 1.5e-3; the test checks
that margin on the oracle's scores before comparing. Bounds as in the
per-block parity tests: indices exact; 2e-2 (bf16) / 1e-4 (fp32) max-abs, plus
half a bf16 ulp for outputs stored in bf16. The backward is given the forward
outputs as the oracle stores them (o rounded to the storage dtype, lse fp32).
"""
import numpy as np
import pytest
import torch

from gated_block_sparse_b200 import inputs, sas
from oracle import sas_oracle as O
from test_gpu_parity import TOL, excess, half_ulp_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gap(scores, k):
    g = np.inf
    for s in scores.values():
        if len(s) > k:
            ss = np.sort(s)[::-1]
            g = min(g, ss[k - 1] - ss[k])
    return g


def _np(t):
    return t.detach().cpu().double().numpy()


@pytest.mark.parametrize("dtype,Hq,Hkv,N,d,topk,seed", [
    ("f32", 2, 2, 640, 64, 2, 31),       # CUDA-core kernels
    ("bf16", 8, 2, 1000, 128, 5, 32),    # tensor-core kernels (bf16, d = 128, even group)
    ("bf16", 4, 2, 2200, 128, 7, 37),    # tensor-core kernels, unions over two mask words
])
def test_tokens_selection_forward_backward(dtype, Hq, Hkv, N, d, topk, seed):
    x = inputs.gen_prefill(1, Hq, Hkv, N, d, dtype, seed=seed, plant="ramp", q_shift=4.0)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "do"))
    ks = sas.sas_block_summary(k)
    idx, cnt, logg = sas.sas_select_tokens(q, ks, Hkv, topk)
    torch.cuda.synchronize()
    oi, oc, ol, scores = O.select_prefill_tokens(x["q"], O.block_summary(x["k"]), Hkv, topk)
    assert _gap(scores, topk) >= 1.5e-3
    assert np.array_equal(idx.cpu().numpy(), oi) and np.array_equal(cnt.cpu().numpy(), oc)
    assert np.abs(_np(logg) - ol).max() < 1e-4
    o, lse = sas.sas_attn_fwd_tokens(q, k, v, idx, cnt, logg)
    torch.cuda.synchronize()
    ol32 = ol.astype(np.float32)
    oo, olse = O.attn_fwd_tokens(x["q"], x["k"], x["v"], oi, oc, ol32)
    o_st = inputs.to_storage(oo, dtype)  # the forward's output as stored
    lse_st = torch.from_numpy(olse.astype(np.float32))
    dq, dk, dv, dlogg = sas.sas_attn_bwd_tokens(q, k, v, o_st.to(DEV), do, lse_st.to(DEV), idx,
                                                cnt, logg)
    torch.cuda.synchronize()
    rq, rk, rv, rdl = O.attn_bwd_tokens(x["q"], x["k"], x["v"], x["do"], oi, oc, ol32,
                                        o_stored=o_st.double().numpy())
    tol = TOL[dtype]
    bf = dtype == "bf16"
    for name, got, ref, stored_bf16 in (("o", o, oo, bf), ("lse", lse, olse, False),
                                        ("dq", dq, rq, bf), ("dk", dk, rk, bf), ("dv", dv, rv, bf),
                                        ("dlogg", dlogg, rdl, False)):
        err = excess(_np(got), ref, tol, stored_bf16, name)
        assert err <= 0, (name, err)
    st, msg = sas.sas_device_status()
    assert st == 0, msg


@pytest.mark.parametrize("dtype,d,Hq,Hkv", [("f32", 64, 2, 1), ("bf16", 128, 4, 2)])
def test_tokens_reduce_to_block_rows_when_rows_agree(dtype, d, Hq, Hkv):
    """Rows of a query block with equal queries select alike: the per-token
    forward and backward equal the per-block ones on the same (repeated)
    selection (fp32: CUDA-core kernels, within rounding; bf16, d = 128: the
    tensor-core kernels, whose per-token units are then the block's own kept
    blocks, bit for bit)."""
    N, topk = 512, 2
    x = inputs.gen_prefill(1, Hq, Hkv, N, d, dtype, seed=34, plant="ramp", q_shift=4.0)
    q = x["q"].clone()
    for t in range(N // 64):
        q[:, :, t * 64:(t + 1) * 64] = q[:, :, t * 64:t * 64 + 1]
    q, k, v, do = q.to(DEV), x["k"].to(DEV), x["v"].to(DEV), x["do"].to(DEV)
    ks = sas.sas_block_summary(k)
    bi, bc, bl = sas.sas_select(q, ks, Hkv, topk, "prefill")
    ti, tc, tl = sas.sas_select_tokens(q, ks, Hkv, topk)
    torch.cuda.synchronize()
    for i in range(N):
        assert torch.equal(ti[:, :, i], bi[:, :, i // 64])
    # the attention calls get the block rows repeated for their 64 tokens, so
    # both see the same gates
    ti, tc, tl = (x_.repeat_interleave(64, dim=2).contiguous() for x_ in (bi, bc, bl))
    ob, lb = sas.sas_attn_fwd(q, k, v, bi, bc, bl)
    ot, lt = sas.sas_attn_fwd_tokens(q, k, v, ti, tc, tl)
    gb = sas.sas_attn_bwd(q, k, v, ob, do, lb, bi, bc, bl)
    gt = sas.sas_attn_bwd_tokens(q, k, v, ob, do, lb, ti, tc, tl)
    torch.cuda.synchronize()
    if dtype == "bf16":
        assert torch.equal(ob, ot) and torch.equal(lb, lt) and torch.equal(gb[0], gt[0])
        # dk, dv sum fp32 partials in L2 in any order, so two runs may round to
        # neighbouring bf16 values: at most one ulp apart
        for a, b in zip(gb[1:3], gt[1:3]):
            a_, b_ = _np(a), _np(b)
            assert np.all(np.abs(a_ - b_) <= 2 * half_ulp_bf16(np.maximum(np.abs(a_), np.abs(b_))))
    else:
        assert float((ob - ot).abs().max()) < 1e-5 and float((lb - lt).abs().max()) < 1e-5
        for a, b in zip(gb[:3], gt[:3]):
            assert float((a - b).abs().max()) < 1e-5
    # the block's dlogg slot is the sum of its tokens' slots
    dl_tok = gt[3].view(1, Hkv, N // 64, 64, topk).sum(dim=3)
    assert float((dl_tok - gb[3]).abs().max()) < 1e-3 * float(gb[3].abs().max()) + 1e-4
    st, msg = sas.sas_device_status()
    assert st == 0, msg


@pytest.mark.parametrize("dtype,Hq,Hkv,N,d,topk,seed", [
    ("f32", 4, 2, 700, 64, 3, 35),
    ("bf16", 8, 2, 4200, 128, 5, 36),   # up to 64 history blocks: two score chunks per block
])
def test_tokens_selector_backward(dtype, Hq, Hkv, N, d, topk, seed):
    """Eq. 8 through per-token selection rows: the selector's share of dq and
    dk, added in place into nonzero gradients, against the oracle on the same
    selection (the GPU's, checked equal to the oracle's first)."""
    x = inputs.gen_prefill(1, Hq, Hkv, N, d, dtype, seed=seed, plant="ramp", q_shift=4.0)
    q, k = x["q"].to(DEV), x["k"].to(DEV)
    ks = sas.sas_block_summary(k)
    idx, cnt, logg = sas.sas_select_tokens(q, ks, Hkv, topk)
    torch.cuda.synchronize()
    oi, oc, _, scores = O.select_prefill_tokens(x["q"], O.block_summary(x["k"]), Hkv, topk)
    assert _gap(scores, topk) >= 1.5e-3
    assert np.array_equal(idx.cpu().numpy(), oi) and np.array_equal(cnt.cpu().numpy(), oc)
    rng = np.random.Generator(np.random.PCG64(seed + 9))
    dl = rng.standard_normal(oi.shape).astype(np.float32)
    dl[oi < 0] = 0.0  # padding slots carry no gradient
    g0 = torch.Generator().manual_seed(seed)
    st = torch.bfloat16 if dtype == "bf16" else torch.float32
    dq0 = (torch.randn(q.shape, generator=g0) * 1e-2).to(st)
    dk0 = (torch.randn(k.shape, generator=g0) * 1e-2).to(st)
    dq, dk = dq0.to(DEV), dk0.to(DEV)
    sas.sas_select_bwd_tokens(q, ks, Hkv, idx, cnt, torch.from_numpy(dl).to(DEV), dq, dk)
    torch.cuda.synchronize()
    st_, msg = sas.sas_device_status()
    assert st_ == 0, msg
    rq, rk = O.select_backward_tokens(x["q"], x["k"], oi, oc, dl, Hkv)
    for name, got, init, ref in (("dq", dq, dq0, rq), ("dk", dk, dk0, rk)):
        want = init.double().numpy() + ref
        g = _np(got)
        if dtype == "f32":  # fp32 accumulation: relative error at fp32 level
            assert np.abs(g - want).max() <= 1e-5 * np.abs(want).max() + 1e-7, name
        else:  # one bf16 rounding of the sum, plus the absolute bound
            assert excess(g, want, TOL["bf16"], True, name) <= 0, name
