"""CPU fp64 oracle for fine-grained top-K sparse attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It restates the method from the pages'
definitions in plain C (``sa_oracle.c``, every value a double) and marshals
numpy arrays to it.  It imports nothing from the CUDA package and the CUDA
package imports nothing from it; both take their inputs from ``workloads``.

Functions (each cites the passage it follows in ``sa_oracle.c``):

``indexer``           I[t,s] = sum_j w[t,j] ReLU(qI[t,j].kI[s]), s <= lim[t]
``e4m3_encode`` / ``e4m3_decode`` / ``indexer_fp8``  the FP8 operand format
``topk``              K best scores per row, ties -> lower position, ascending
``pool_mean``         mean of each complete block of index keys
``two_stage``         coarse block top-k, then fine top-K inside the blocks
``page_selection``    whole kept blocks (+ own block), no fine pass
``selection``         S(t) = TopK(t) U {max(0,t-W+1) .. t}
``sparse_attention``  softmax(q.k * scale) v over S(t)
``prefill`` / ``decode``  the three stages end to end

Parity is pinned by tests/test_oracle_pins.py (closed forms, brute force,
the pages' dense and masked attention formulas).
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from workloads import bf16_to_f64, unpage

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_i64p = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile sa_oracle.c with gcc (strict IEEE double, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off",
                               "-fno-fast-math", "-fPIC", "-shared", "-o", tmp,
                               _SRC, "-lpthread", "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32 = ctypes.c_int64, ctypes.c_int
        lib.oracle_indexer.argtypes = [i64, i32, i32, i32, _f64p, _f64p, _f64p, _i64p, _f64p, i32]
        _u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
        lib.oracle_e4m3_encode.argtypes = [i64, _f64p, _u8p]
        lib.oracle_e4m3_decode.argtypes = [i64, _u8p, _f64p]
        lib.oracle_topk.argtypes = [i64, i64, _f64p, _i64p, ctypes.c_void_p, i32, _i64p, i32]
        lib.oracle_pool_mean.argtypes = [i64, i32, i32, _f64p, _f64p]
        lib.oracle_two_stage.argtypes = [i64, _i64p, i32, i32, _f64p, _f64p, i64, _f64p,
                                         i32, i32, i32, _i64p, _i64p, i32]
        lib.oracle_selection.argtypes = [i32, _i64p, i32, i64, _i64p]
        lib.oracle_selection.restype = i64
        lib.oracle_sparse_attention.argtypes = [i64, i32, i32, _f64p, _f64p, _f64p, _i64p,
                                                _i64p, ctypes.c_double, _f64p, ctypes.c_void_p, i32]
        _lib = lib
    return _lib


def threads() -> int:
    return int(os.environ.get("ORACLE_THREADS", os.cpu_count() or 1))


def _f64(x) -> np.ndarray:
    """bf16 bits (uint16) are widened exactly; anything else is cast."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return bf16_to_f64(x)
    return np.ascontiguousarray(x, dtype=np.float64)


def _i64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.int64)


# --------------------------------------------------------------------------
# stage 1: indexer
# --------------------------------------------------------------------------
def indexer(qI, w, kI, lim, S=None) -> np.ndarray:
    """Scores [R, S]: column s <= lim[r] holds the indexer score, others -inf."""
    qI, w, kI, lim = _f64(qI), _f64(w), _f64(kI), _i64(lim)
    R, H, D = qI.shape
    S = kI.shape[0] if S is None else S
    assert kI.shape[0] >= S and w.shape == (R, H) and lim.shape == (R,)
    out = np.empty((R, S), dtype=np.float64)
    _load().oracle_indexer(R, S, H, D, qI.reshape(-1), w.reshape(-1),
                           np.ascontiguousarray(kI[:S]).reshape(-1), lim, out, threads())
    return out


def e4m3_encode(x) -> np.ndarray:
    """Nearest OCP e4m3 code of each value (ties to even, +-448 saturation)."""
    x = _f64(x)
    out = np.empty(x.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode(x.size, np.ascontiguousarray(x).reshape(-1), out.reshape(-1))
    return out


def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 code (uint8) as a double."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    _load().oracle_e4m3_decode(codes.size, codes.reshape(-1), out.reshape(-1))
    return out


def indexer_fp8(qI_codes, w, kI_codes, lim, S=None) -> np.ndarray:
    """The indexer over e4m3 operands: the same scores computed on the values
    the codes hold (the FP8 indexer quantises its operands, nothing else)."""
    return indexer(e4m3_decode(qI_codes), w, e4m3_decode(kI_codes), lim, S)


# --------------------------------------------------------------------------
# stage 2: top-K and selection set
# --------------------------------------------------------------------------
def topk(scores, n_valid, K, cand=None) -> np.ndarray:
    """Top-K positions per row among columns [0, n_valid[r]) (positions are the
    columns, or cand[r, col]); ties -> lower position; ascending; -1 padded."""
    scores = _f64(scores)
    R, L = scores.shape
    n_valid = _i64(n_valid)
    out = np.empty((R, K), dtype=np.int64)
    cand_arr = None if cand is None else _i64(cand)
    if cand_arr is not None:
        assert cand_arr.shape == (R, L)
    ptr = None if cand_arr is None else cand_arr.ctypes.data_as(ctypes.c_void_p)
    _load().oracle_topk(R, L, scores, n_valid, ptr, K, out, threads())
    return out


def pool_mean(kI, blk) -> np.ndarray:
    kI = _f64(kI)
    S, D = kI.shape
    out = np.empty((S // blk, D), dtype=np.float64)
    _load().oracle_pool_mean(S, D, blk, kI.reshape(-1), out.reshape(-1) if out.size else np.empty(1))
    return out


def two_stage(t_pos, qI, w, kI, blk, keep, K):
    """Coarse block top-`keep`, then fine top-K among the kept blocks' tokens
    plus the query's own block.  Returns (topk [R,K], blocks [R,keep])."""
    t_pos, qI, w, kI = _i64(t_pos), _f64(qI), _f64(w), _f64(kI)
    R, H, D = qI.shape
    topk_out = np.empty((R, K), dtype=np.int64)
    blocks = np.empty((R, keep), dtype=np.int64)
    _load().oracle_two_stage(R, t_pos, H, D, qI.reshape(-1), w.reshape(-1), kI.shape[0],
                             kI.reshape(-1), blk, keep, K, topk_out, blocks, threads())
    return topk_out, blocks


def page_selection(t_pos, qI, w, kI, blk, keep):
    """Page-granular selection: whole blocks instead of single tokens (the
    64-token page selection of "Sparse Attention" (completesystemdesign.dev),
    DSA list, and the block routing of "Sparse Attention in 2026", "The
    designs that shipped").  The coarse pass keeps `keep` blocks, and the
    selection is every token of those blocks plus the query's own block up to
    t, with no fine pass.  That is the two-stage selection whose fine top-K
    may keep all keep*blk + blk candidates, so it is computed as such.
    Returns (positions [R, keep*blk + blk] ascending, -1 padded; blocks)."""
    return two_stage(t_pos, qI, w, kI, blk, keep, keep * blk + blk)


def selection(topk_rows, W, t_pos):
    """CSR (ptr, idx) of S(t) = TopK(t) U Window(t), each row sorted, unique."""
    topk_rows, t_pos = _i64(topk_rows), _i64(t_pos)
    R, K = topk_rows.shape
    lib = _load()
    buf = np.empty(K + W, dtype=np.int64)
    ptr = np.zeros(R + 1, dtype=np.int64)
    parts = []
    for r in range(R):
        n = lib.oracle_selection(K, np.ascontiguousarray(topk_rows[r]), W, int(t_pos[r]), buf)
        parts.append(buf[:n].copy())
        ptr[r + 1] = ptr[r] + n
    idx = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    return ptr, np.ascontiguousarray(idx, dtype=np.int64)


# --------------------------------------------------------------------------
# stage 3: exact attention over the selection
# --------------------------------------------------------------------------
def sparse_attention(q, k, v, sel_ptr, sel_idx, scale):
    """(out [R,Hq,d], lse [R,Hq]) over the CSR key sets."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    R, Hq, d = q.shape
    out = np.empty((R, Hq, d), dtype=np.float64)
    lse = np.empty((R, Hq), dtype=np.float64)
    sel_idx = _i64(sel_idx) if len(sel_idx) else np.zeros(1, dtype=np.int64)
    _load().oracle_sparse_attention(R, Hq, d, q.reshape(-1), k.reshape(-1), v.reshape(-1),
                                    _i64(sel_ptr), sel_idx, float(scale), out,
                                    lse.ctypes.data_as(ctypes.c_void_p), threads())
    return out, lse


# --------------------------------------------------------------------------
# end to end
# --------------------------------------------------------------------------
def prefill(inp: dict, K: int, W: int, rows=None, block=None, keep=None):
    """The three stages for the query rows `rows` (default: all) of one causal
    sequence.  With `block`/`keep` the selection is the two-stage one.
    Returns dict(topk, sel_ptr, sel_idx, out, lse[, blocks])."""
    N = inp["q"].shape[0]
    rows = np.arange(N, dtype=np.int64) if rows is None else _i64(rows)
    res = {}
    if block is None:
        sc = indexer(inp["qI"][rows], inp["w"][rows], inp["kI"], rows, S=N)
        res["topk"] = topk(sc, rows + 1, K)
    else:
        res["topk"], res["blocks"] = two_stage(rows, inp["qI"][rows], inp["w"][rows],
                                               inp["kI"], block, keep, K)
    ptr, idx = selection(res["topk"], W, rows)
    d = inp["q"].shape[2]
    res["out"], res["lse"] = sparse_attention(inp["q"][rows], inp["k"], inp["v"], ptr, idx,
                                              1.0 / np.sqrt(d))
    res["sel_ptr"], res["sel_idx"] = ptr, idx
    return res


def decode_sequence(inp: dict, b: int):
    """Logical (unpaged) k, v, kI of sequence b of a decode input."""
    L = int(inp["lengths"][b])
    if "page_table" in inp:
        tbl = inp["page_table"][b]
        return (unpage(inp["k"], tbl, L), unpage(inp["v"], tbl, L),
                unpage(inp["kI"], tbl, L))
    return inp["k"][b, :L], inp["v"][b, :L], inp["kI"][b, :L]


def decode(inp: dict, K: int, W: int, seqs=None):
    """One query per sequence at position len_b - 1.
    Returns dict(topk [B,K], out [B,Hq,d], lse [B,Hq], n_sel [B])."""
    B = inp["q"].shape[0]
    seqs = range(B) if seqs is None else seqs
    d = inp["q"].shape[2]
    tk, outs, lses, nsel = [], [], [], []
    for b in seqs:
        k, v, kI = decode_sequence(inp, b)
        t = np.array([k.shape[0] - 1], dtype=np.int64)
        sc = indexer(inp["qI"][b:b + 1], inp["w"][b:b + 1], kI, t)
        top = topk(sc, t + 1, K)
        ptr, idx = selection(top, W, t)
        o, l = sparse_attention(inp["q"][b:b + 1], k, v, ptr, idx, 1.0 / np.sqrt(d))
        tk.append(top[0]); outs.append(o[0]); lses.append(l[0]); nsel.append(ptr[1])
    return dict(topk=np.stack(tk), out=np.stack(outs), lse=np.stack(lses),
                n_sel=np.array(nsel))
