"""Seeded synthetic inputs for fine-grained top-K sparse attention.

This module only *draws data*: it holds none of the method's arithmetic, so
both the CPU oracle (``oracle/``) and the CUDA path (``fine_grained_top_b200``)
may use it without sharing any part of the computation.

Recipe (the same for every workload):

* q, k, v  ~ N(0, 1) drawn in float32 and rounded to bf16 (round to nearest
  even);
* qI, kI   ~ U{-3, ..., 3} and w ~ U{0, ..., 3}, integers stored as bf16, so
  every indexer score is an exact integer in fp32 (max 8 * 3 * 64 * 9 < 2**24);
* one ``numpy.random.Generator(PCG64)`` stream per tensor, spawned from
  ``SeedSequence(seed)`` in the fixed order
  q, k, v, qI, kI, w, lengths, page permutation;
* paged caches hold 64-token pages; each sequence's pages are a random
  permutation of the pool's pages (the page table is padded with -1).

All bf16 tensors are returned as ``numpy.uint16`` arrays of raw bf16 bits.
"""

from __future__ import annotations

import numpy as np

STREAMS = ("q", "k", "v", "qI", "kI", "w", "lengths", "perm")

# The workloads, named by what they are.  Shapes follow the pages'
# long-context regimes: 8K-128K prefill, 128K-class decode, top-k 2048 and
# 64-token KV pages.
CONFIGS = {
    "prefill_512": dict(kind="prefill", N=512, Hq=4, d=64, H_I=2, D_I=32,
                        K=64, W=32),
    "prefill_8k": dict(kind="prefill", N=8192, Hq=16, d=128, H_I=4, D_I=64,
                       K=1024, W=128),
    "decode_8x128k": dict(kind="decode", B=8, L=131072, Hq=64, d=128, H_I=8,
                          D_I=64, K=2048, W=512, paged=False),
    "prefill_64k_two_stage": dict(kind="two_stage", N=65536, Hq=16, d=128,
                                  H_I=4, D_I=64, block=64, keep=64, K=2048,
                                  W=512),
    # the 64K two-stage shapes on a 16K sequence: a case small enough for
    # multi-pass profiler captures of the same kernels
    "prefill_16k_two_stage": dict(kind="two_stage", N=16384, Hq=16, d=128,
                                  H_I=4, D_I=64, block=64, keep=64, K=2048,
                                  W=512),
    "decode_paged_16x256k": dict(kind="decode", B=16, L_min=16384,
                                 L_max=262144, page=64, Hq=64, d=128, H_I=8,
                                 D_I=64, K=2048, W=512, paged=True),
}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return raw bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + 0x7FFF + ((b >> 16) & 1)
    return (b >> 16).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits to float64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def _streams(seed: int) -> dict:
    children = np.random.SeedSequence(seed).spawn(len(STREAMS))
    return {name: np.random.Generator(np.random.PCG64(c))
            for name, c in zip(STREAMS, children)}


def _normal_bf16(rng, shape) -> np.ndarray:
    return bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def _int_bf16(rng, lo, hi, shape) -> np.ndarray:
    return bf16_bits(rng.integers(lo, hi + 1, size=shape).astype(np.float32))


def gen_prefill(N: int, Hq: int, d: int, H_I: int, D_I: int, seed: int = 0,
                **_ignored) -> dict:
    """One causal sequence of N tokens (query t sits at position t)."""
    r = _streams(seed)
    return dict(
        q=_normal_bf16(r["q"], (N, Hq, d)),
        k=_normal_bf16(r["k"], (N, d)),
        v=_normal_bf16(r["v"], (N, d)),
        qI=_int_bf16(r["qI"], -3, 3, (N, H_I, D_I)),
        kI=_int_bf16(r["kI"], -3, 3, (N, D_I)),
        w=_int_bf16(r["w"], 0, 3, (N, H_I)),
    )


def gen_decode(B: int, Hq: int, d: int, H_I: int, D_I: int, *, L: int = None,
               L_min: int = None, L_max: int = None, lengths=None,
               paged: bool = False, page: int = 64, seed: int = 0,
               **_ignored) -> dict:
    """B sequences with one new query each, at position len_b - 1.

    Contiguous caches are [B, L_max, *]; paged caches are pools
    [P, page, *] addressed through page_table[B, max_pages].
    """
    r = _streams(seed)
    if lengths is None:
        if L is not None:
            lengths = np.full(B, L, dtype=np.int32)
        else:
            lengths = r["lengths"].integers(L_min, L_max + 1, size=B).astype(np.int32)
    lengths = np.asarray(lengths, dtype=np.int32)
    out = dict(lengths=lengths,
               q=_normal_bf16(r["q"], (B, Hq, d)),
               qI=_int_bf16(r["qI"], -3, 3, (B, H_I, D_I)),
               w=_int_bf16(r["w"], 0, 3, (B, H_I)))
    if not paged:
        S = int(lengths.max())
        out.update(k=_normal_bf16(r["k"], (B, S, d)),
                   v=_normal_bf16(r["v"], (B, S, d)),
                   kI=_int_bf16(r["kI"], -3, 3, (B, S, D_I)))
        return out
    n_pages = (lengths + page - 1) // page
    P = int(n_pages.sum())
    max_pages = int(n_pages.max())
    perm = r["perm"].permutation(P).astype(np.int32)
    table = np.full((B, max_pages), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, :n_pages[b]] = perm[off:off + n_pages[b]]
        off += n_pages[b]
    out.update(page_table=table, page=page,
               k=_normal_bf16(r["k"], (P, page, d)),
               v=_normal_bf16(r["v"], (P, page, d)),
               kI=_int_bf16(r["kI"], -3, 3, (P, page, D_I)))
    return out


def unpage(pool: np.ndarray, table_row: np.ndarray, length: int) -> np.ndarray:
    """Logical [length, *] view of one sequence of a paged pool (a copy)."""
    page = pool.shape[1]
    n = (length + page - 1) // page
    rows = pool[table_row[:n]].reshape(n * page, *pool.shape[2:])
    return rows[:length]


def config_inputs(name: str, seed: int = 0) -> dict:
    cfg = CONFIGS[name]
    if cfg["kind"] in ("prefill", "two_stage"):
        return gen_prefill(seed=seed, **cfg)
    return gen_decode(seed=seed, **cfg)
