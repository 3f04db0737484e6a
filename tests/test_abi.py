"""The C-ABI library builds, loads without a GPU, exports every function
include/bi.h declares, and rejects bad arguments on the host (these checks
return before any CUDA call)."""
import ctypes

import pytest

from helpers import header_functions


@pytest.fixture(scope="module")
def libbi():
    from invariant_bi_lora_b200 import build, bi
    build.build()
    return bi.lib()


def test_exports_every_declared_symbol(libbi):
    names = header_functions()
    assert len(names) >= 18, names
    missing = [n for n in names if not hasattr(libbi, n)]
    assert not missing, missing


def test_binding_covers_header(libbi):
    from invariant_bi_lora_b200 import bi
    assert set(header_functions()) == set(bi._SIGS), set(header_functions()) ^ set(bi._SIGS)


def test_status_strings(libbi):
    from invariant_bi_lora_b200 import bi
    for code, name in bi.STATUS_NAMES.items():
        assert bi.status_string(code) == name
    assert bi.status_string(99) == "BI_ERR_UNKNOWN"


def test_sizes(libbi):
    from invariant_bi_lora_b200 import bi
    from helpers import plan_words
    # perm 4096 + offsets 10 + 2 words of padding + 73 records of 68 words
    assert bi.lora_plan_bytes(4096, 8) == 4 * (4096 + 10 + 2 + 68 * 73) == 4 * plan_words(4096, 8)
    assert bi.lora_plan_bytes(0, 1) == 4 * (4 + 68 * 2) == 4 * plan_words(0, 1)
    assert bi.lora_plan_bytes(1000, 256) == 4 * plan_words(1000, 256)


FAKE = ctypes.c_void_p(0x10000)   # never dereferenced: every call below fails validation


@pytest.mark.parametrize("M,K,r,splits,mode,want", [
    (16, 100, 16, 8, 2, 2),      # K not a multiple of the 64-wide leaf
    (16, 4096, 12, 8, 2, 2),     # r not a multiple of 8
    (16, 4096, 16, 3, 2, 2),     # splits not a power of two
    (16, 4096, 16, 32, 2, 2),    # more splits than a cluster holds
    (16, 128, 16, 4, 2, 2),      # splits does not divide the 2 leaves
    (16, 4096, 16, 8, 0, 2),     # UNSPLIT takes splits = 1
    (16, 4096, 16, 8, 7, 1),     # unknown mode
    (-1, 4096, 16, 8, 2, 1),     # negative M
])
def test_shrink_rejects(libbi, M, K, r, splits, mode, want):
    st = libbi.bi_lora_shrink(FAKE, FAKE, FAKE, M, K, r, splits, mode, None)
    assert st == want


def test_other_rejects(libbi):
    assert libbi.bi_lora_shrink(None, None, None, 0, 4096, 16, 8, 2, None) == 0    # M == 0: no-op
    assert libbi.bi_lora_shrink(ctypes.c_void_p(0x10001), FAKE, FAKE, 4, 64, 8, 1, 0, None) == 2  # misaligned
    assert libbi.bi_lora_plan(FAKE, 16, 0, FAKE, 1 << 20, None) == 1
    assert libbi.bi_lora_plan(FAKE, 16, 8, FAKE, 8, None) == 3                   # plan too small
    assert libbi.bi_lora_plan(FAKE, 16, 8, ctypes.c_void_p(0x10004), 1 << 20, None) == 2   # not 16-byte aligned
    assert libbi.bi_lora_expand(FAKE, FAKE, FAKE, 4, 12, 64, 0, None) == 2
    assert libbi.bi_rmsnorm(FAKE, FAKE, FAKE, 4, 100, ctypes.c_float(1e-6), None) == 2
    assert libbi.bi_log_softmax(FAKE, FAKE, 4, 6, None) == 2
    assert libbi.bi_mean(FAKE, FAKE, -1, 8, None) == 1
    assert libbi.bi_tree_combine(FAKE, FAKE, 0, 16, None) == 1
    assert libbi.bi_tree_combine(FAKE, FAKE, 65, 16, None) == 1
    ptrs2 = (ctypes.c_void_p * 2)(FAKE, FAKE)
    assert libbi.bi_tree_combine_peers(ptrs2, 0, FAKE, 0, 16, None) == 1            # s < 1
    assert libbi.bi_tree_combine_peers(ptrs2, 65, FAKE, 0, 16, None) == 1           # s > 64
    assert libbi.bi_tree_combine_peers(None, 2, FAKE, 0, 16, None) == 1             # no pointer array
    assert libbi.bi_tree_combine_peers(ptrs2, 2, FAKE, 2, 16, None) == 2            # begin not a multiple of 4
    bad = (ctypes.c_void_p * 2)(FAKE, ctypes.c_void_p(0x10004))
    assert libbi.bi_tree_combine_peers(bad, 2, FAKE, 0, 16, None) == 2              # a partial misaligned
    nul = (ctypes.c_void_p * 2)(FAKE, None)
    assert libbi.bi_tree_combine_peers(nul, 2, FAKE, 0, 16, None) == 1              # a null partial
    assert libbi.bi_tree_combine_peers(ptrs2, 2, FAKE, 0, 0, None) == 0             # empty range: no-op
    assert libbi.bi_math_spec(FAKE, FAKE, 16, 4, None) == 1
    assert libbi.bi_selftest_bounded_wait(0, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from invariant_bi_lora_b200 import bi
    monkeypatch.setattr(bi, "_lib", None)
    monkeypatch.setattr(bi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        bi.lib()
