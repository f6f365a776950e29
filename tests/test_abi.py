"""The C ABI loads, exports every entry point include/sas.h declares, and
rejects bad arguments on the host before any launch (CPU only: no call here
reaches a kernel)."""
import ctypes
import os
import re

import pytest

from gated_block_sparse_b200 import sas

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sas.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sas_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from gated_block_sparse_b200 import build
    build.build()
    return sas.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) == 32
    for n in names:
        assert hasattr(lib, n), n
        assert n in sas.SIGNATURES, n


def test_strerror_and_version(lib):
    assert lib.sas_version() == 100
    for code, text in [(0, b"ok"), (1, b"invalid argument"), (2, b"unsupported configuration"),
                       (3, b"CUDA error"), (4, b"device wait timed out"), (5, b"internal error")]:
        assert lib.sas_strerror(code) == text


def test_workspace_sizes_are_consistent(lib):
    # the one-launch decode needs no workspace; the split decode attention does
    assert lib.sas_decode_workspace_size(8, 32, 8, 131072, 128, 31) == 0
    a = lib.sas_decode_attend_workspace_size(1, 32, 8, 65536, 128, 15)
    b = lib.sas_decode_attend_workspace_size(8, 32, 8, 131072, 128, 31)
    assert a > 0 and b > a and a % 16 == 0 and b % 16 == 0
    # prefill selection needs one fp32 query summary per (b, group, block)
    assert lib.sas_select_workspace_size(1, 32, 8, 16384, 128, 31, 0) == 8 * 256 * 128 * 4
    assert lib.sas_attn_bwd_workspace_size(1, 32, 8, 16384, 128, 31, 1) == 2 * 8 * 16384 * 128 * 4
    assert lib.sas_decode_attend_workspace_size(0, 32, 8, 65536, 128, 15) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def test_rejects_bad_head_dim(lib):
    st = lib.sas_block_summary(FAKE, 1, 1, 2, 128, 96, None, FAKE, None)
    assert st == 2 and b"head dim" in lib.sas_last_error_message()


def test_rejects_group_mismatch(lib):
    st = lib.sas_attn_fwd(FAKE, FAKE, FAKE, 1, 1, 6, 4, 128, 64, FAKE, FAKE, FAKE, 2, 0.0, FAKE,
                          FAKE, None, 0, None)
    assert st == 1 and b"multiple" in lib.sas_last_error_message()


def test_rejects_null_and_misaligned_pointers(lib):
    st = lib.sas_attn_fwd(None, FAKE, FAKE, 1, 1, 4, 4, 128, 64, FAKE, FAKE, FAKE, 2, 0.0, FAKE,
                          FAKE, None, 0, None)
    assert st == 1 and b"q must not be NULL" in lib.sas_last_error_message()
    st = lib.sas_attn_fwd(FAKE + 4, FAKE, FAKE, 1, 1, 4, 4, 128, 64, FAKE, FAKE, FAKE, 2, 0.0,
                          FAKE, FAKE, None, 0, None)
    assert st == 1 and b"aligned" in lib.sas_last_error_message()


def test_rejects_topk_and_workspace(lib):
    st = lib.sas_select(FAKE, 1, FAKE, 1, 4, 4, 128, 64, 129, 0, None, 0.0, FAKE, FAKE, FAKE,
                        None, FAKE, 1 << 20, None)
    assert st == 2
    st = lib.sas_select(FAKE, 1, FAKE, 1, 4, 4, 128, 64, 2, 0, None, 0.0, FAKE, FAKE, FAKE,
                        None, FAKE, 16, None)
    assert st == 1 and b"workspace too small" in lib.sas_last_error_message()
    # the optional raw-score output, when given, must be aligned like every other buffer
    st = lib.sas_select(FAKE, 1, FAKE, 1, 4, 4, 128, 64, 2, 0, None, 0.0, FAKE, FAKE, FAKE,
                        FAKE + 4, FAKE, 1 << 20, None)
    assert st == 1 and b"scores_out" in lib.sas_last_error_message()


def test_rejects_bad_decode_shapes(lib):
    ws = 1 << 20
    st = lib.sas_decode(FAKE, FAKE, FAKE, 1, 1, 24, 8, 65536, 128, FAKE, FAKE, 15, 1, 0.0, FAKE,
                        None, FAKE, ws, None)
    assert st == 2  # 3 query heads per kv head is not a supported group size
    st = lib.sas_decode(FAKE, FAKE, FAKE, 1, 1, 32, 8, 65000, 128, FAKE, FAKE, 15, 1, 0.0, FAKE,
                        None, FAKE, ws, None)
    assert st == 1 and b"multiple of 64" in lib.sas_last_error_message()
    st = lib.sas_decode(FAKE, FAKE, FAKE, 1, 1, 32, 8, 65536, 128, FAKE, FAKE, 15, 2, 0.0, FAKE,
                        None, FAKE, ws, None)
    assert st == 1 and b"gated" in lib.sas_last_error_message()



def test_rejects_bad_summary_dtype(lib):
    st = lib.sas_block_summary_ex(FAKE, 1, 1, 8, 1024, 128, None, FAKE, 7, None)
    assert st == 1 and b"summary dtype" in lib.sas_last_error_message()
    st = lib.sas_decode_ex(FAKE, FAKE, FAKE, 1, 1, 32, 8, 65536, 128, FAKE, FAKE, 7, 15, 1, 0.0,
                           FAKE, None, None)
    assert st == 1 and b"summary dtype" in lib.sas_last_error_message()
    st = lib.sas_decode_paged_ex(FAKE, FAKE, FAKE, FAKE, 7, 1, 1, 32, 8, 16, 128, FAKE, 16, FAKE,
                                 15, 1, 0.0, FAKE, None, None)
    assert st == 1 and b"summary dtype" in lib.sas_last_error_message()

def test_summary_upkeep_argument_checks(lib):
    st = lib.sas_block_summary_last(FAKE, 1, 1, 8, 1000, 128, FAKE, FAKE, 0, None, 0, None)
    assert st == 1 and b"multiple of 64" in lib.sas_last_error_message()
    st = lib.sas_block_summary_last(FAKE, 1, 1, 8, 1024, 128, FAKE, FAKE, 0, FAKE, 0, None)
    assert st == 1 and b"npages" in lib.sas_last_error_message()
    st = lib.sas_block_summary_last(FAKE, 1, 1, 8, 1024, 128, FAKE, FAKE, 3, None, 0, None)
    assert st == 1 and b"summary dtype" in lib.sas_last_error_message()
    st = lib.sas_block_summary_last(FAKE, 1, 1, 8, 1024, 96, FAKE, FAKE, 0, None, 0, None)
    assert st == 2  # head dim 96 is not supported
    assert lib.sas_block_summary_last(None, 1, 0, 8, 1024, 128, None, None, 0, None, 0, None) == 0

def test_empty_inputs_are_noops(lib):
    # B = 0 or N = 0: nothing to do, no pointer needed, no launch
    assert lib.sas_attn_fwd(None, None, None, 1, 0, 4, 4, 128, 64, None, None, None, 2, 0.0, None,
                            None, None, 0, None) == 0
    assert lib.sas_block_summary(None, 1, 1, 2, 63, 64, None, None, None) == 0


def test_noalloc_selection_capacity_and_rejection(lib):
    assert lib.sas_select_prefill_noalloc_capacity() == 4 << 20
    # 8 groups x 2048 query blocks x 128 x 4 B = 8 MiB of query summaries: rejected before launch
    st = lib.sas_select_prefill_noalloc(FAKE, 1, FAKE, 1, 8, 8, 131072, 128, 4, 0.0, FAKE, FAKE,
                                        FAKE, None)
    assert st == 2 and b"exceed" in lib.sas_last_error_message()
