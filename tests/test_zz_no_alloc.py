"""The no-allocation prefill selection (sas_select_prefill_noalloc) against
the workspace version (sas_select in prefill mode).

sas_select_prefill_noalloc serves callers that may not allocate device
memory when they call into the library, for example a host runtime that hands
the library only its input and output buffers: its scratch is a fixed device
array inside libsas instead of a caller workspace. This checks, through the
C ABI, that two calls in a row (different shapes, so the second reuses
memory the first left behind) give the same indices and counts as
sas_select and as the fp64 oracle, and log gates within the suite's fp32
bound of both; and that after a first call (which looks up the array's
address once) further calls leave the device's free memory unchanged.

Kept in a file that pytest collects last, so a run stopped at its first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
import numpy as np
import pytest
import torch

from gated_block_sparse_b200 import inputs, sas
from oracle import sas_oracle as O

pytestmark = pytest.mark.gpu


def _case(B, Hq, Hkv, N, d, topk, seed):
    x = inputs.gen_prefill(B, Hq, Hkv, N, d, "bf16", seed=seed, plant="ramp")
    q, k = x["q"].cuda(), x["k"].cuda()
    ks = sas.sas_block_summary(k)
    return q, ks, Hkv, topk, x


def test_noalloc_selection_matches_workspace_version_twice():
    cases = [_case(1, 32, 8, 16384, 128, 31, seed=901),   # 1 MiB of query summaries
             _case(2, 8, 2, 3000, 64, 5, seed=902)]       # smaller second call
    for q, ks, Hkv, topk, x in cases:
        ref = sas.sas_select(q, ks, Hkv, topk, "prefill")
        got = sas.sas_select_prefill_noalloc(q, ks, Hkv, topk)
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
        assert float((got[2] - ref[2]).abs().max()) <= 1e-4
        oi, oc, ol, _ = O.select_prefill(x["q"], O.block_summary(x["k"]), Hkv, topk)
        assert np.array_equal(got[0].cpu().numpy(), oi) and np.array_equal(got[1].cpu().numpy(), oc)
        assert np.abs(got[2].cpu().double().numpy() - ol).max() <= 1e-4


def test_noalloc_calls_leave_free_device_memory_unchanged():
    q, ks, Hkv, topk, _ = _case(1, 16, 4, 8192, 128, 15, seed=903)
    T = q.shape[2] // 64
    out = (torch.empty((1, Hkv, T, topk), dtype=torch.int32, device="cuda"),
           torch.empty((1, Hkv, T), dtype=torch.int32, device="cuda"),
           torch.empty((1, Hkv, T, topk), dtype=torch.float32, device="cuda"))
    sas.sas_select_prefill_noalloc(q, ks, Hkv, topk, out=out)  # first call: address lookup
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        sas.sas_select_prefill_noalloc(q, ks, Hkv, topk, out=out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_rejects_problems_beyond_the_fixed_array():
    lib = sas.load_library()
    cap = lib.sas_select_prefill_noalloc_capacity()
    assert cap == 4 << 20
    q = torch.empty((1, 8, 64, 128), dtype=torch.bfloat16, device="cuda")
    ks = torch.empty((8, 1, 128), dtype=torch.float32, device="cuda")
    idx = torch.empty((8, 1, 1), dtype=torch.int32, device="cuda")
    st = lib.sas_select_prefill_noalloc(q.data_ptr(), 1, ks.data_ptr(), 1, 8, 8, 8192 * 16, 128,
                                        1, 0.0, idx.data_ptr(), idx.data_ptr(), ks.data_ptr(),
                                        None)
    assert st == 2 and b"exceed" in lib.sas_last_error_message()
