"""bench.py host logic on CPU: the clock record taken around a timed region."""
import importlib.util
import os
import tempfile
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _sampler(bench, lines):
    f = tempfile.NamedTemporaryFile("w", suffix=".csv", delete=False)
    f.write("".join(lines))
    f.close()
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.f = open(f.name)
    return c


def _t(stamp):
    return time.mktime(time.strptime(stamp, "%Y/%m/%d %H:%M:%S"))


ROW = "2026/12/02 10:00:0{s}.100, {mhz}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, {cap}\n"


def test_clock_summary_inside_the_window():
    b = _bench()
    c = _sampler(b, [ROW.format(s=s, mhz=m, cap="Not Active") for s, m in ((1, 1900), (2, 1965), (3, 1965))]
                 + [ROW.format(s=4, mhz=1800, cap="Active")])
    got = c.summary(_t("2026/12/02 10:00:02"), _t("2026/12/02 10:00:03"))
    assert got["sm_mhz"] == 1965.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == [] and got["samples"] == 2


def test_clock_summary_region_shorter_than_the_sampling_period():
    """A timed region that no sample falls in takes the next sample, else the
    last one (a region of a few ms, as a 2-step prefill run)."""
    b = _bench()
    c = _sampler(b, [ROW.format(s=1, mhz=1965, cap="Active")])
    got = c.summary(_t("2026/12/02 10:00:05"), _t("2026/12/02 10:00:05") + 0.006)
    assert got["sm_mhz"] == 1965.0 and got["reasons"] == ["sw_power_cap"] and got["samples"] == 1


def test_clock_summary_without_samples():
    b = _bench()
    c = _sampler(b, [])
    got = c.summary(0.0, 1.0)
    assert got["sm_mhz"] is None and got["reasons"] == ["no nvidia-smi samples"]


def test_decode_byte_accounting_matches_the_stated_figures():
    """c2: 4,194,304 B of kept K/V (15 blocks + a full current block, 8 kv
    heads), 4,190,208 B of fp32 summaries (1023 blocks), q and o 8 KB each;
    c5: 16,777,216 B of K/V and 33,550,336 B of summaries (half with bf16)."""
    from gated_block_sparse_b200 import inputs
    b = _bench()
    c2 = inputs.CONFIGS["c2"]
    sel, att, step = b.decode_bytes(c2, [65536])
    assert sel == 4190208 + 8192 and att == 4194304 + 2 * 8192 and step == 8400896
    c5 = inputs.CONFIGS["c5"]
    sel, att, step = b.decode_bytes(c5, [524288])
    assert sel - 8192 == 33550336 and att - 16384 == 16777216
    sel16, _, step16 = b.decode_bytes(c5, [524288], "bf16")
    assert sel16 - 8192 == 33550336 // 2 and step - step16 == 33550336 // 2
    # a ragged row: C = 1, kk = 1, current block of 1 token
    c = dict(c2, B=1)
    sel, att, step = b.decode_bytes(c, [65])
    assert att == 8 * (64 + 1) * 128 * 2 * 2 + 2 * 8192 and sel == 8 * 1 * 128 * 4 + 8192


def test_prefill_flop_accounting_closed_form():
    """c3 with every query block keeping min(t, 31) history blocks: per head,
    sum_t 64 * 64 * min(t, 31) kept pairs plus 64 * 65 / 2 causal pairs of the
    current block; 4 d FLOPs per pair forward, 10 d backward. These are the
    0.508 / 1.270 TFLOP figures the c3 record is quoted on."""
    import numpy as np
    b = _bench()
    N, Hq, Hkv, d, T = 16384, 32, 8, 128, 256
    cnt = np.minimum(np.arange(T), 31)[None, None, :].repeat(Hkv, axis=1)
    f, bw = b.prefill_flops(cnt, N, Hq, Hkv, d)
    pairs = Hq * (sum(64 * 64 * min(t, 31) for t in range(T)) + T * 64 * 65 // 2)
    assert f == 4 * d * pairs and bw == 10 * d * pairs
    assert f == 508014100480 and bw == 1270035251200
    # a ragged last block of 8 rows sees 8 * 64 keys per kept block and 8 * 9 / 2 causal pairs
    f2, _ = b.prefill_flops(np.array([[[0, 1]]]), 72, 2, 1, 64)
    assert f2 == 4 * 64 * 2 * (64 * 65 // 2 + 8 * 64 + 8 * 9 // 2)


def test_prefill_flop_accounting_per_token_rows():
    """Per-token rows: token i of a head sees 64 keys per kept block and the
    i % 64 + 1 causal keys of its own block."""
    import numpy as np
    b = _bench()
    cnt = np.array([[[0] * 64 + [1] * 64 + [2] * 64]])  # B = 1, Hkv = 1, N = 192
    f, bw = b.prefill_flops_tokens(cnt, 192, 4, 1, 64)
    pairs = 4 * (64 * (64 * 1 + 64 * 2) + 3 * (64 * 65 // 2))
    assert f == 4 * 64 * pairs and bw == 10 * 64 * pairs


def test_reference_arm_times_exactly_k_steps():
    """--impl reference: W untimed and K timed oracle steps, each a bounded
    sample (here one query-block unit of the tiny prefill workload)."""
    b = _bench()
    got = b.reference_arm("c1", "f32", 3, 1)
    assert got["steps"] == 3 and got["warmup"] == 1
    assert got["value"] > 0 and got["unit"] == "TFLOP/s"
    assert got["cpu_baseline"]["kind"] == "oracle" and got["cpu_baseline"]["cores"] == 1
