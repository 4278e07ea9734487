"""The C-ABI library loads and exports every symbol include/sa.h declares.

CPU only: nothing here launches a kernel.  The argument checks exercised
return before the library touches a device.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sa.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^SA_API [^(]*?\b(sa_\w+)\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    import prompt_aware_head_b200 as pkg
    return pkg


def test_header_declares_the_boundary_calls():
    names = _declared()
    for must in ("sa_build_layout", "sa_select_blocks", "sa_block_sparse_attention", "sa_pattern_mask",
                 "sa_dense_attention", "sa_density"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for name in _declared():
        assert hasattr(so, name), name
    assert set(_declared()) == set(lib.EXPORTED)


def test_status_strings_and_version(lib):
    assert lib.sa_status_string(lib.SA_OK) == "ok"
    assert "head" in lib.sa_status_string(lib.SA_ERR_HEAD_MASK)
    assert "sm_100a" in lib.sa_version()


def test_budget_matches_reading(lib):
    # clamp(floor(rho * C + 1e-4), 1, C) for the five workloads' budgets
    assert lib.sa_budget(0.5, 6) == 3
    assert [lib.sa_budget(r, 64) for r in (0.3, 0.5, 1.0)] == [19, 32, 64]
    assert lib.sa_budget(0.3, 256) == 76
    assert lib.sa_budget(0.2, 512) == 102
    assert lib.sa_budget(0.7, 10) == 7
    assert lib.sa_budget(0.001, 64) == 1


def test_workspace_size_and_shape_errors(lib):
    n = lib.sa_workspace_size(1, 24, 16896, 128)
    assert n > 24 * 264 * 128 * 4 * 2
    with pytest.raises(lib.SAError) as e:
        lib.sa_workspace_size(1, 24, 16900, 128)   # N not a multiple of 64
    assert e.value.status == lib.SA_ERR_SHAPE
    with pytest.raises(lib.SAError):
        lib.sa_workspace_size(1, 24, 4096, 96)     # d not 64 / 128


def test_argument_checks_before_any_launch(lib):
    fake = 1 << 20  # aligned, never dereferenced: the checks fail first
    with pytest.raises(lib.SAError) as e:
        lib.sa_dense_attention(fake, fake, fake, 1, 4, 512, 32, 0.0, fake, fake, 1 << 20, stream=0)
    assert e.value.status == lib.SA_ERR_SHAPE
    with pytest.raises(lib.SAError) as e:
        lib.sa_block_sparse_attention(fake, fake, fake, 1, 4, 512, 64, fake, fake, 8, [1, 0, 0, 0], 4, 0.0, fake,
                                      fake, 1 << 30, stream=0)
    assert e.value.status == lib.SA_ERR_HEAD_MASK
    with pytest.raises(lib.SAError) as e:
        lib.sa_block_sparse_attention(fake + 2, fake, fake, 1, 4, 512, 64, fake, fake, 8, None, 0, 0.0, fake,
                                      fake, 1 << 30, stream=0)
    assert e.value.status == lib.SA_ERR_INVALID_ARG     # misaligned Q
    with pytest.raises(lib.SAError) as e:
        lib.sa_block_sparse_attention(fake, fake, fake, 1, 4, 512, 64, fake, fake, 8, None, 0, 0.0, fake, fake, 16,
                                      stream=0)
    assert e.value.status == lib.SA_ERR_WORKSPACE
    with pytest.raises(lib.SAError) as e:
        lib.sa_block_sparse_attention(fake, fake, fake, 1, 4, 512, 64, fake, fake, 8, None, 0, -1.0, fake,
                                      fake, 1 << 30, stream=0)
    assert e.value.status == lib.SA_ERR_INVALID_ARG     # negative softmax scale


def test_grouped_head_counts_checked_before_any_launch(lib):
    fake = 1 << 20
    for H_kv in (0, 4, 12):  # 6 query heads: no key heads, a partial group, more key than query heads
        with pytest.raises(lib.SAError) as e:
            lib.sa_dense_attention_gqa(fake, fake, fake, 1, 6, H_kv, 512, 64, 0.0, fake, fake, 1 << 20, stream=0)
        assert e.value.status == lib.SA_ERR_SHAPE
        with pytest.raises(lib.SAError) as e:
            lib.sa_block_sparse_attention_gqa(fake, fake, fake, 1, 6, H_kv, 512, 64, fake, fake, 8, None, 0, 0.0,
                                              fake, fake, 1 << 30, stream=0)
        assert e.value.status == lib.SA_ERR_SHAPE


def test_binding_constants_match_the_crate(lib):
    from tests.conftest import read_golden
    g = read_golden("crate_constants.txt")
    assert lib.MIN_ACTIVE_HEADS == int(g["MIN_ACTIVE_HEADS"])
    assert lib.DEFAULT_SPARSITY == float(g["DEFAULT_SPARSITY"])
    assert lib.MAX_QUALITY_LOSS == float(g["MAX_QUALITY_LOSS"])
