"""The C-ABI library loads on a CPU-only machine, exports every symbol that
include/sa.h declares, and rejects bad arguments synchronously (these checks
run before any CUDA call, so no GPU is needed)."""

import ctypes
import os
import re

import pytest

from tests.conftest import ROOT


@pytest.fixture(scope="module")
def sa():
    import __graft_entry__
    __graft_entry__.build()
    import fine_grained_top_b200 as m
    return m


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "sa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sa_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(sa):
    names = _declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(sa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sa.SIGNATURES)


def test_no_dynamic_cuda_runtime_or_driver_dependency(sa):
    # loads without libcuda/libcudart: cudart is static, the driver is reached lazily
    import subprocess
    out = subprocess.run(["ldd", sa.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out and "libcuda.so" not in out


def test_status_strings_and_version(sa):
    lib = sa._lib
    assert lib.sa_status_string(0) == b"SA_OK"
    assert lib.sa_status_string(6) == b"SA_ERR_WORKSPACE"
    assert sa.sa_version() == 101
    assert sa.sa_dev_status_decode(0) == sa.SA_OK
    assert sa.sa_dev_status_decode(sa.SA_DEV_INDEX) == sa.SA_ERR_INDEX
    assert sa.sa_dev_status_decode(sa.SA_DEV_ORDER) == sa.SA_ERR_INDEX
    assert sa.sa_dev_status_decode(sa.SA_DEV_TIMEOUT | sa.SA_DEV_INDEX) == sa.SA_ERR_TIMEOUT


P = ctypes.c_void_p(16)   # a fake, 16-byte aligned, never dereferenced pointer
N0 = None


def test_topk_blocks_argument_checks(sa):
    f = sa._lib.sa_topk_select_blocks
    # scores, ld, T, S, blocks, keep, block, K, topk, dev_status, stream
    assert f(P, 4160, 10, 9, P, 64, 64, 2048, P, N0, N0) == sa.SA_ERR_INVALID_ARG      # S < T
    assert f(P, 4100, 10, 10, P, 64, 64, 2048, P, N0, N0) == sa.SA_ERR_INVALID_ARG     # ld < keep*block + block
    assert f(P, 4162, 10, 10, P, 64, 64, 2048, P, N0, N0) == sa.SA_ERR_INVALID_ARG     # ld not a multiple of 4
    assert f(P, 524352, 10, 10, P, 8192, 64, 2048, P, N0, N0) == sa.SA_ERR_UNSUPPORTED  # rows of 524352 columns
    assert f(P, 4160, 10, 10, N0, 64, 64, 2048, P, N0, N0) == sa.SA_ERR_INVALID_ARG    # no block ids
    assert f(ctypes.c_void_p(20), 4160, 10, 10, P, 64, 64, 2048, P, N0, N0) == sa.SA_ERR_INVALID_ARG   # misaligned
    assert f(P, 4160, 0, 10, P, 64, 64, 2048, P, N0, N0) == sa.SA_OK                   # nothing to do
    assert f(P, 64, 10, 10, N0, 0, 64, 0, P, N0, N0) == sa.SA_OK                       # K = 0


def test_fused_indexer_topk_decode_argument_checks(sa):
    f = sa._lib.sa_indexer_topk_decode
    # qI, w, kI, page_table, max_pages, pool_pages, page_size, B, S, H_I, D_I, seq_lens, K, topk, dev_status, stream
    assert f(P, P, P, N0, 0, 0, 64, -1, 1024, 8, 64, P, 64, P, N0, N0) == sa.SA_ERR_INVALID_ARG     # B < 0
    assert f(P, P, P, N0, 0, 0, 64, 2, 1024, 9, 64, P, 64, P, N0, N0) == sa.SA_ERR_UNSUPPORTED      # H_I > 8
    assert f(P, P, P, N0, 0, 0, 64, 2, 1024, 8, 32, P, 64, P, N0, N0) == sa.SA_ERR_UNSUPPORTED      # D_I = 32
    assert f(P, P, P, N0, 0, 0, 64, 2, 600000, 8, 64, P, 64, P, N0, N0) == sa.SA_ERR_UNSUPPORTED    # S too long
    assert f(P, P, P, P, 16, 10, 32, 2, 1024, 8, 64, P, 64, P, N0, N0) == sa.SA_ERR_UNSUPPORTED     # page_size 32
    assert f(P, P, P, P, 8, 10, 64, 2, 1024, 8, 64, P, 64, P, N0, N0) == sa.SA_ERR_INVALID_ARG      # 8 pages < S
    assert f(P, P, P, P, 16, 0, 64, 2, 1024, 8, 64, P, 64, P, N0, N0) == sa.SA_ERR_INVALID_ARG      # empty pool
    assert f(P, P, N0, N0, 0, 0, 64, 2, 1024, 8, 64, P, 64, P, N0, N0) == sa.SA_ERR_INVALID_ARG     # no keys
    assert f(P, P, ctypes.c_void_p(24), N0, 0, 0, 64, 2, 1024, 8, 64, P, 64, P, N0, N0) == sa.SA_ERR_INVALID_ARG
    assert f(P, P, P, N0, 0, 0, 64, 0, 1024, 8, 64, P, 64, P, N0, N0) == sa.SA_OK                    # nothing to do
    assert f(P, P, P, N0, 0, 0, 64, 2, 1024, 8, 64, P, 0, P, N0, N0) == sa.SA_OK                     # K = 0


def test_topk_argument_checks(sa):
    f = sa._lib.sa_topk_select
    assert f(P, 8, -1, 8, N0, N0, 0, 4, P, N0, N0) == sa.SA_ERR_INVALID_ARG      # rows < 0
    assert f(P, 6, 2, 8, N0, N0, 0, 4, P, N0, N0) == sa.SA_ERR_INVALID_ARG       # ld < row_len
    assert f(P, 10, 2, 8, N0, N0, 0, 4, P, N0, N0) == sa.SA_ERR_INVALID_ARG      # ld not multiple of 4
    assert f(N0, 8, 2, 8, N0, N0, 0, 4, P, N0, N0) == sa.SA_ERR_INVALID_ARG      # NULL scores
    assert f(ctypes.c_void_p(20), 8, 2, 8, N0, N0, 0, 4, P, N0, N0) == sa.SA_ERR_INVALID_ARG  # misaligned
    assert f(P, 8, 2, 8, N0, P, 4, 4, P, N0, N0) == sa.SA_ERR_INVALID_ARG        # ld_cand < row_len
    assert f(P, 600000, 2, 600000, N0, N0, 0, 4, P, N0, N0) == sa.SA_ERR_UNSUPPORTED   # > 16 x 32768
    assert f(P, 8, 0, 8, N0, N0, 0, 4, P, N0, N0) == sa.SA_OK                    # nothing to do
    assert f(P, 8, 2, 8, N0, N0, 0, 0, P, N0, N0) == sa.SA_OK                    # K = 0


def test_indexer_argument_checks(sa):
    f = sa._lib.sa_indexer_scores
    ok = dict(H=4, D=64)
    assert f(P, P, P, N0, 0, 0, 64, 1, 8, 8, 4, 48, N0, P, 8, N0, N0) == sa.SA_ERR_UNSUPPORTED  # D_I
    assert f(P, P, P, N0, 0, 0, 64, 1, 8, 8, 3, 64, N0, P, 8, N0, N0) == sa.SA_ERR_UNSUPPORTED  # H_I
    assert f(P, P, P, N0, 0, 0, 64, 1, 8, 8, 4, 64, N0, P, 4, N0, N0) == sa.SA_ERR_INVALID_ARG  # ld < S
    assert f(P, P, P, N0, 0, 0, 64, 1, 9, 8, 4, 64, N0, P, 8, N0, N0) == sa.SA_ERR_INVALID_ARG  # T > S causal
    assert f(P, P, P, P, 1, 4, 32, 1, 1, 8, 4, 64, P, P, 8, N0, N0) == sa.SA_ERR_UNSUPPORTED   # page 32
    assert f(P, P, P, P, 1, 4, 64, 1, 1, 128, 4, 64, P, P, 128, N0, N0) == sa.SA_ERR_INVALID_ARG  # pages short
    assert f(N0, P, P, N0, 0, 0, 64, 1, 8, 8, 4, 64, N0, P, 8, N0, N0) == sa.SA_ERR_INVALID_ARG
    assert f(P, P, P, N0, 0, 0, 64, 0, 8, 8, 4, 64, N0, P, 8, N0, N0) == sa.SA_OK
    assert ok


def test_indexer_fp8_and_convert_argument_checks(sa):
    f = sa._lib.sa_indexer_scores_fp8
    assert f(P, P, P, N0, 0, 0, 64, 1, 8, 8, 4, 32, N0, P, 8, N0, N0) == sa.SA_ERR_UNSUPPORTED  # D_I 32
    assert f(P, P, P, N0, 0, 0, 64, 1, 8, 8, 3, 64, N0, P, 8, N0, N0) == sa.SA_ERR_UNSUPPORTED  # H_I
    assert f(P, P, P, N0, 0, 0, 64, 1, 8, 8, 4, 128, N0, P, 4, N0, N0) == sa.SA_ERR_INVALID_ARG  # ld < S
    assert f(P, P, ctypes.c_void_p(24), N0, 0, 0, 64, 1, 8, 8, 4, 64, N0, P, 8, N0, N0) \
        == sa.SA_ERR_INVALID_ARG   # kI not 16-byte aligned
    assert f(P, P, P, N0, 0, 0, 64, 1, 8, 0, 4, 128, N0, P, 8, N0, N0) == sa.SA_OK  # S = 0
    g = sa._lib.sa_convert_e4m3
    assert g(P, P, -1, N0) == sa.SA_ERR_INVALID_ARG
    assert g(N0, P, 5, N0) == sa.SA_ERR_INVALID_ARG
    assert g(N0, N0, 0, N0) == sa.SA_OK


def test_attention_argument_checks(sa):
    f = sa._lib.sa_sparse_attn_prefill
    assert f(P, P, P, P, 4, 2, 8, 8, 16, 96, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_ERR_UNSUPPORTED   # d = 96
    assert f(P, P, P, P, 4, 2, 8, 8, 65, 128, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_ERR_UNSUPPORTED  # Hq > 64
    assert f(P, P, P, P, 4, 2, 9, 8, 16, 128, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_ERR_INVALID_ARG  # T > S
    assert f(P, P, P, N0, 4, 2, 8, 8, 16, 128, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_ERR_INVALID_ARG  # NULL topk
    assert f(P, P, P, P, -1, 2, 8, 8, 16, 128, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_ERR_INVALID_ARG
    assert f(P, P, P, P, 4, 2, 8, 8, 16, 128, 0.1, P, N0, P, 1024, N0, N0) == sa.SA_ERR_INVALID_ARG  # ws align
    assert sa.sa_prefill_workspace_bytes(8192, 8192, 1024, 128, 16, 128) == 8192 * 256 * 4
    assert sa.sa_prefill_workspace_bytes(65536, 65536, 2048, 512, 16, 128) == 0       # sparse: gathered path
    assert f(P, P, P, P, 4, 2, 0, 8, 16, 128, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_OK
    assert f(P, P, P, P, 0, 0, 8, 8, 16, 128, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_ERR_INVALID_ARG  # empty key sets
    assert f(P, P, P, P, 0, 0, 0, 8, 16, 128, 0.1, P, N0, N0, 0, N0, N0) == sa.SA_OK               # no queries
    g = sa._lib.sa_sparse_attn_decode
    need = sa.sa_decode_workspace_bytes(8, 64, 128, 2048, 512)
    assert need > 8 * 64 * 128 * 4
    W = ctypes.c_void_p(256)
    assert g(P, P, P, N0, 0, 0, 64, 100, P, P, 2048, 512, 8, 64, 128, 0.1, P, N0, W, need - 1, N0, N0) \
        == sa.SA_ERR_WORKSPACE
    assert g(P, P, P, N0, 0, 0, 64, 100, P, P, 2048, 512, 8, 64, 128, 0.1, P, N0, P, need, N0, N0) \
        == sa.SA_ERR_INVALID_ARG   # workspace not 256-byte aligned
    assert g(P, P, P, P, 0, 1, 64, 100, P, P, 2048, 512, 8, 64, 128, 0.1, P, N0, W, need, N0, N0) \
        == sa.SA_ERR_INVALID_ARG   # paged without pages


def test_two_stage_helper_checks(sa):
    lib = sa._lib
    assert lib.sa_expand_blocks(P, 8, 8, 4, 64, P, 100, P, N0, N0) == sa.SA_ERR_INVALID_ARG   # ld_cand small
    assert lib.sa_pool_index_keys(P, 128, 48, 64, P, N0) == sa.SA_ERR_UNSUPPORTED
    assert lib.sa_pool_index_keys(P, 63, 64, 64, P, N0) == sa.SA_OK                         # no full block
    assert lib.sa_coarse_block_counts(9, 8, 64, P, N0) == sa.SA_ERR_INVALID_ARG


def test_selftest_argument_checks(sa):
    lib = sa._lib
    assert lib.sa_selftest_wait_timeout(0, P, N0) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_selftest_wait_timeout(100, N0, N0) == sa.SA_ERR_INVALID_ARG
