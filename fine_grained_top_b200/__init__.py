"""B200-native fine-grained top-K sparse attention.

The compute lives in ``libsa.so`` (C ABI, ``include/sa.h``): hand-written
CUDA for sm_100a.  This module only marshals arguments to it: every entry
point below has the name and the argument order of its C counterpart, takes
torch tensors for device buffers (PyTorch supplies memory and streams), and
raises ``SAError`` when the library returns a non-OK status.  There is no
Python or CPU fallback: importing fails loudly if the library is missing.

``pipeline`` builds the three-stage step (indexer -> top-K -> sparse
attention) out of these calls with preallocated buffers.
"""

from __future__ import annotations

import ctypes
import os

# SA_LIBRARY may name another build of the same library (e.g. a tuning variant)
LIB_PATH = os.environ.get("SA_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsa.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_CUDA = 0, 1, 2, 3
SA_ERR_TIMEOUT, SA_ERR_INDEX, SA_ERR_WORKSPACE = 4, 5, 6
SA_DEV_INDEX, SA_DEV_ORDER, SA_DEV_TIMEOUT = 0x1, 0x2, 0x4

# Every symbol include/sa.h declares, with its ctypes signature.
_vp, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "sa_status_string": (ctypes.c_char_p, [_i32]),
    "sa_dev_status_decode": (_i32, [_i32]),
    "sa_version": (_i32, []),
    "sa_indexer_scores": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                 _vp, _vp, _i64, _vp, _vp]),
    "sa_indexer_scores_fp8": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                     _vp, _vp, _i64, _vp, _vp]),
    "sa_convert_e4m3": (_i32, [_vp, _vp, _i64, _vp]),
    "sa_indexer_scores_candidates": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp,
                                            _i64, _vp, _vp]),
    "sa_block_scores_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "sa_indexer_scores_blocks": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _i32, _i32, _vp, _i64,
                                        _vp, _sz, _vp, _vp]),
    "sa_topk_select": (_i32, [_vp, _i64, _i32, _i32, _vp, _vp, _i64, _i32, _vp, _vp, _vp]),
    "sa_topk_select_blocks": (_i32, [_vp, _i64, _i32, _i32, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "sa_indexer_topk_decode": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _i32,
                                      _vp, _vp, _vp]),
    "sa_prefill_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "sa_sparse_attn_prefill": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp,
                                      _vp, _vp, _sz, _vp, _vp]),
    "sa_decode_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "sa_sparse_attn_decode": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _i32,
                                     _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz, _vp, _vp]),
    "sa_sparse_attn_decode_noalloc": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _i32,
                                             _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _vp]),
    "sa_pool_index_keys": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "sa_coarse_block_counts": (_i32, [_i32, _i32, _i32, _vp, _vp]),
    "sa_expand_blocks": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _i64, _vp, _vp, _vp]),
    "sa_selftest_wait_timeout": (_i32, [_i32, _vp, _vp]),
}


class SAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s returned %s" % (where, _lib.sa_status_string(status).decode()))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libsa.so is not built; run `python fine_grained_top_b200/build.py` "
                          "(there is no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def _ptr(t):
    """Device (or host) address of a tensor; None -> NULL."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libsa must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, where):
    if status != SA_OK:
        raise SAError(status, where)


# ---------------------------------------------------------------- entry points
def sa_indexer_scores(qI, w, kI, page_table, max_pages, pool_pages, page_size, B, T, S, H_I, D_I,
                      n_valid, scores, ld_scores, dev_status=None, stream=None):
    _check(_lib.sa_indexer_scores(_ptr(qI), _ptr(w), _ptr(kI), _ptr(page_table), max_pages, pool_pages,
                                  page_size, B, T, S, H_I, D_I, _ptr(n_valid), _ptr(scores), ld_scores,
                                  _ptr(dev_status), _stream(stream)), "sa_indexer_scores")


def sa_indexer_scores_fp8(qI, w, kI, page_table, max_pages, pool_pages, page_size, B, T, S, H_I, D_I,
                          n_valid, scores, ld_scores, dev_status=None, stream=None):
    """qI, kI: uint8 tensors of e4m3 bits (see sa_convert_e4m3)."""
    _check(_lib.sa_indexer_scores_fp8(_ptr(qI), _ptr(w), _ptr(kI), _ptr(page_table), max_pages, pool_pages,
                                      page_size, B, T, S, H_I, D_I, _ptr(n_valid), _ptr(scores), ld_scores,
                                      _ptr(dev_status), _stream(stream)), "sa_indexer_scores_fp8")


def sa_convert_e4m3(src, dst, n, stream=None):
    _check(_lib.sa_convert_e4m3(_ptr(src), _ptr(dst), n, _stream(stream)), "sa_convert_e4m3")


def sa_indexer_scores_candidates(qI, w, kI, T, S, H_I, D_I, cand, ld_cand, n_cand, scores, ld_scores,
                                 dev_status=None, stream=None):
    _check(_lib.sa_indexer_scores_candidates(_ptr(qI), _ptr(w), _ptr(kI), T, S, H_I, D_I, _ptr(cand),
                                             ld_cand, _ptr(n_cand), _ptr(scores), ld_scores,
                                             _ptr(dev_status), _stream(stream)),
           "sa_indexer_scores_candidates")


def sa_block_scores_workspace_bytes(T, S, keep) -> int:
    return int(_lib.sa_block_scores_workspace_bytes(T, S, keep))


def sa_indexer_scores_blocks(qI, w, kI, T, S, H_I, D_I, blocks, keep, block, scores, ld_scores, workspace,
                             workspace_bytes, dev_status=None, stream=None):
    _check(_lib.sa_indexer_scores_blocks(_ptr(qI), _ptr(w), _ptr(kI), T, S, H_I, D_I, _ptr(blocks), keep, block,
                                         _ptr(scores), ld_scores, _ptr(workspace), workspace_bytes,
                                         _ptr(dev_status), _stream(stream)), "sa_indexer_scores_blocks")


def sa_topk_select(scores, ld_scores, rows, row_len, n_valid, cand_map, ld_cand, K, topk,
                   dev_status=None, stream=None):
    _check(_lib.sa_topk_select(_ptr(scores), ld_scores, rows, row_len, _ptr(n_valid), _ptr(cand_map),
                               ld_cand, K, _ptr(topk), _ptr(dev_status), _stream(stream)), "sa_topk_select")


def sa_topk_select_blocks(scores, ld_scores, T, S, blocks, keep, block, K, topk, dev_status=None, stream=None):
    _check(_lib.sa_topk_select_blocks(_ptr(scores), ld_scores, T, S, _ptr(blocks), keep, block, K, _ptr(topk),
                                      _ptr(dev_status), _stream(stream)), "sa_topk_select_blocks")


def sa_indexer_topk_decode(qI, w, kI, page_table, max_pages, pool_pages, page_size, B, S, H_I, D_I, seq_lens, K,
                           topk, dev_status=None, stream=None):
    _check(_lib.sa_indexer_topk_decode(_ptr(qI), _ptr(w), _ptr(kI), _ptr(page_table), max_pages, pool_pages,
                                       page_size, B, S, H_I, D_I, _ptr(seq_lens), K, _ptr(topk),
                                       _ptr(dev_status), _stream(stream)), "sa_indexer_topk_decode")


def sa_prefill_workspace_bytes(T, S, K, W, Hq, d) -> int:
    return int(_lib.sa_prefill_workspace_bytes(T, S, K, W, Hq, d))


def sa_sparse_attn_prefill(q, k, v, topk, K, W, T, S, Hq, d, scale, out, lse=None, workspace=None,
                           workspace_bytes=0, dev_status=None, stream=None):
    _check(_lib.sa_sparse_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(topk), K, W, T, S, Hq, d,
                                       float(scale), _ptr(out), _ptr(lse), _ptr(workspace), int(workspace_bytes),
                                       _ptr(dev_status), _stream(stream)), "sa_sparse_attn_prefill")


def sa_decode_workspace_bytes(B, Hq, d, K, W) -> int:
    return int(_lib.sa_decode_workspace_bytes(B, Hq, d, K, W))


def sa_sparse_attn_decode(q, k_cache, v_cache, page_table, max_pages, pool_pages, page_size, S_max, seq_lens,
                          topk, K, W, B, Hq, d, scale, out, lse, workspace, workspace_bytes,
                          dev_status=None, stream=None):
    _check(_lib.sa_sparse_attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table), max_pages,
                                      pool_pages, page_size, S_max, _ptr(seq_lens), _ptr(topk), K, W, B,
                                      Hq, d, float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                      workspace_bytes, _ptr(dev_status), _stream(stream)),
           "sa_sparse_attn_decode")


def sa_sparse_attn_decode_noalloc(q, k_cache, v_cache, page_table, max_pages, pool_pages, page_size, S_max,
                                  seq_lens, topk, K, W, B, Hq, d, scale, out, lse=None, dev_status=None,
                                  stream=None):
    """Decode for callers that cannot allocate device memory: the split partials
    go to a fixed 16 MiB array inside the library instead of a workspace.
    Concurrent calls on one GPU share that array and must not overlap."""
    _check(_lib.sa_sparse_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                              max_pages, pool_pages, page_size, S_max, _ptr(seq_lens),
                                              _ptr(topk), K, W, B, Hq, d, float(scale), _ptr(out), _ptr(lse),
                                              _ptr(dev_status), _stream(stream)),
           "sa_sparse_attn_decode_noalloc")


SA_DECODE_NOALLOC_SCRATCH_BYTES = 16 << 20


def sa_pool_index_keys(kI, S, D_I, block, kB, stream=None):
    _check(_lib.sa_pool_index_keys(_ptr(kI), S, D_I, block, _ptr(kB), _stream(stream)), "sa_pool_index_keys")


def sa_coarse_block_counts(T, S, block, n_blocks, stream=None):
    _check(_lib.sa_coarse_block_counts(T, S, block, _ptr(n_blocks), _stream(stream)), "sa_coarse_block_counts")


def sa_expand_blocks(blocks, T, S, keep, block, cand, ld_cand, n_cand, dev_status=None, stream=None):
    _check(_lib.sa_expand_blocks(_ptr(blocks), T, S, keep, block, _ptr(cand), ld_cand, _ptr(n_cand),
                                 _ptr(dev_status), _stream(stream)), "sa_expand_blocks")


def sa_dev_status_decode(word: int) -> int:
    return int(_lib.sa_dev_status_decode(int(word)))


def sa_version() -> int:
    return int(_lib.sa_version())


def sa_selftest_wait_timeout(limit_us, dev_status, stream=None):
    _check(_lib.sa_selftest_wait_timeout(int(limit_us), _ptr(dev_status), _stream(stream)),
           "sa_selftest_wait_timeout")
