"""Failure detection on the GPU without a fault: the bounded-wait path.

Every device wait of the library gives up after a wall-clock limit and
records a bit in a device error word, which sas_device_status reads back.
The self-test kernel waits on a barrier that nothing completes, so its wait
runs out; the test checks that the status reports the timeout, that clearing
works, and that an ordinary decode step leaves no error behind.
"""
import time

import pytest
import torch

from gated_block_sparse_b200 import inputs, sas

pytestmark = pytest.mark.gpu

SAS_OK, SAS_ERR_TIMEOUT = 0, 4


def test_forced_wait_timeout_is_reported_and_cleared():
    sas.sas_device_status(clear=True)  # start from clean words
    st, _ = sas.sas_device_status()
    assert st == SAS_OK
    t0 = time.perf_counter()
    sas.sas_debug_wait_timeout()
    st, msg = sas.sas_device_status(clear=True)
    dt = time.perf_counter() - t0
    assert st == SAS_ERR_TIMEOUT, (st, msg)
    assert "k_wait_selftest" in msg and "gave up" in msg
    assert 0.15 < dt < 10.0  # the wait limit is 200 ms; the call returned
    st, msg = sas.sas_device_status()
    assert st == SAS_OK, msg
    # the context is still usable: a small decode runs and reports no error
    x = inputs.gen_decode(1, 8, 2, 4096, 128, [3000], "bf16", seed=77, planted=4)
    q, kc, vc, lens = (x[k].cuda() for k in ("q", "kc", "vc", "lens"))
    ks = sas.sas_block_summary(kc)
    o = sas.sas_decode(q, kc, vc, lens, ks, 3)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    st, msg = sas.sas_device_status()
    assert st == SAS_OK, msg
