"""GPU parity: every stage through the C ABI against the CPU fp64 oracle.

Index sets (top-K, block selection, candidates) must match bit for bit;
attention outputs within max-abs 2e-2 and mean-abs 2e-3 of the fp64 result.
Inputs are the seeded synthetic workloads (workloads/); nothing here reads a
stored GPU result.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, bf16_bits, bf16_to_f64, config_inputs, gen_decode, gen_prefill
from tests.gpu_helpers import assert_close_attention, dev, host_f64, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_top_b200 as m
    return m


def _pl():
    from fine_grained_top_b200.pipeline import DecodePlan, PrefillPlan
    return PrefillPlan, DecodePlan


def _to_dev(inp, names=("q", "k", "v", "qI", "w", "kI")):
    return {n: dev(inp[n]) for n in names}


# ====================================================================== top-K
def _scores(rows, L, dist, rng):
    if dist == "ties3":
        return rng.integers(0, 3, size=(rows, L)).astype(np.float32)
    if dist == "ints":
        return rng.integers(0, 2000, size=(rows, L)).astype(np.float32)
    return rng.standard_normal((rows, L)).astype(np.float32)


@pytest.mark.parametrize("rows,L,K,dist", [
    (37, 700, 64, "ties3"), (16, 5000, 1024, "ints"), (50, 17000, 700, "normal"),
    (3, 40000, 100, "normal"), (8, 131072, 2048, "ints"), (4, 262144, 2048, "ties3"),
    (5, 393216, 3000, "ints"), (2, 524288, 2048, "normal"), (9, 33, 40, "normal"), (64, 1023, 64, "ints"),
    (300, 8192, 1024, "ties3"), (33, 16384, 16000, "ties3"),
    # rows of at most 1024 columns (one warp per row)
    (100, 1024, 64, "ties3"), (77, 257, 200, "normal"), (5, 1024, 1023, "ints"), (1000, 1000, 64, "ints"),
    (3, 1, 1, "normal"), (20, 700, 699, "ties3"),
])
def test_topk_matches_oracle(sa, rows, L, K, dist):
    rng = np.random.default_rng(rows * 7 + L)
    sc = _scores(rows, L, dist, rng)
    n_valid = rng.integers(0, L + 1, size=rows).astype(np.int32)
    n_valid[0] = L
    n_valid[-1] = min(L, K)
    if rows > 2:
        n_valid[1] = 0
    ld = (L + 3) // 4 * 4
    buf = np.full((rows, ld), np.nan, np.float32)
    buf[:, :L] = sc
    out = torch.empty((rows, K), dtype=torch.int32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_topk_select(dev(buf), ld, rows, L, dev(n_valid), None, 0, K, out, ds)
    want = oracle.topk(sc.astype(np.float64), n_valid, K)
    assert status(ds) == 0
    assert np.array_equal(out.cpu().numpy(), want)


def test_topk_causal_default_and_neg_inf(sa):
    rng = np.random.default_rng(3)
    rows, L, K = 300, 300, 37
    sc = rng.integers(0, 5, size=(rows, L)).astype(np.float32)
    sc[:, ::7] = -np.inf
    out = torch.empty((rows, K), dtype=torch.int32, device="cuda")
    sa.sa_topk_select(dev(sc), L, rows, L, None, None, 0, K, out)
    want = oracle.topk(sc.astype(np.float64), np.arange(rows) + 1, K)
    assert np.array_equal(out.cpu().numpy(), want)


@pytest.mark.parametrize("rows,L,K", [(40, 4160, 2048), (50, 1000, 64), (33, 300, 100)])
def test_topk_candidate_map(sa, rows, L, K):
    rng = np.random.default_rng(4 + L)
    sc = rng.integers(0, 50, size=(rows, L)).astype(np.float32)
    cand = np.sort(rng.choice(1 << 20, size=(rows, L), replace=True), axis=1).astype(np.int32)
    cand = cand + np.arange(L, dtype=np.int32)[None, :]          # strictly ascending
    n_valid = rng.integers(min(1000, L // 2), L + 1, size=rows).astype(np.int32)
    out = torch.empty((rows, K), dtype=torch.int32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_topk_select(dev(sc), L, rows, L, dev(n_valid), dev(cand), L, K, out, ds)
    want = oracle.topk(sc.astype(np.float64), n_valid, K, cand=cand)
    assert status(ds) == 0
    assert np.array_equal(out.cpu().numpy(), want)


@pytest.mark.parametrize("T,S,keep,K,dist", [(300, 5000, 64, 2048, "ties3"), (257, 4097, 16, 500, "ints"),
                                             (100, 100, 4, 50, "normal"), (130, 9000, 0, 40, "ints"),
                                             (64, 64 * 70, 127, 1000, "ties3")])
def test_topk_over_block_ids_matches_oracle(sa, T, S, keep, K, dist):
    # the two-stage fine select reading its candidates from the kept block ids
    rng = np.random.default_rng(T + keep)
    blk = 64
    pos = np.arange(S - T, S)
    own = pos // blk
    blocks = np.full((T, max(keep, 1)), -1, dtype=np.int32)
    n_kept = np.zeros(T, dtype=np.int64)
    for t in range(T):
        k = min(keep, int(own[t]), int(rng.integers(0, keep + 1)) if t % 3 == 0 else keep)
        blocks[t, :k] = np.sort(rng.choice(int(own[t]), size=k, replace=False)) if k else []
        n_kept[t] = k
    L = keep * blk + blk
    ld = (L + 3) // 4 * 4
    sc = _scores(T, ld, dist, rng)
    # the oracle's view: candidate positions in column order
    cand = np.zeros((T, L), dtype=np.int64)
    for t in range(T):
        toks = (blocks[t, :n_kept[t]][:, None] * blk + np.arange(blk)[None, :]).reshape(-1)
        toks = np.r_[toks, own[t] * blk + np.arange(pos[t] - own[t] * blk + 1)]
        cand[t, :len(toks)] = toks
        cand[t, len(toks):] = toks[-1] + 1 + np.arange(L - len(toks))   # unused columns, ascending
    n_valid = n_kept * blk + (pos - own * blk + 1)
    out = torch.empty((T, K), dtype=torch.int32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_topk_select_blocks(dev(sc), ld, T, S, dev(blocks) if keep else None, keep, blk, K, out, ds)
    want = oracle.topk(sc[:, :L].astype(np.float64), n_valid, K, cand=cand)
    assert status(ds) == 0
    assert np.array_equal(out.cpu().numpy(), want)


def test_topk_over_block_ids_reports_bad_ids(sa):
    T, S, keep, K = 8, 1000, 4, 16
    blocks = np.tile(np.array([0, 1, 2, 3], dtype=np.int32), (T, 1))
    blocks[3, 2] = 999                       # not below the own block
    blocks[5] = [2, 1, 3, 4]                 # not ascending
    sc = np.zeros((T, keep * 64 + 64), dtype=np.float32)
    out = torch.empty((T, K), dtype=torch.int32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_topk_select_blocks(dev(sc), keep * 64 + 64, T, S, dev(blocks), keep, 64, K, out, ds)
    st = status(ds)
    assert st & sa.SA_DEV_INDEX and st & sa.SA_DEV_ORDER


# ====================================================================== indexer
@pytest.mark.parametrize("N,H_I,D_I,rows", [
    (512, 2, 32, None), (1000, 4, 64, None), (300, 8, 64, None), (777, 1, 32, None),
    (129, 4, 64, None), (1, 4, 64, None), (8192, 4, 64, 384),
])
def test_indexer_prefill_exact(sa, N, H_I, D_I, rows):
    inp = gen_prefill(N=N, Hq=1, d=64, H_I=H_I, D_I=D_I, seed=N + H_I)
    t = _to_dev(inp, ("qI", "w", "kI"))
    ld = (N + 3) // 4 * 4
    sc = torch.full((N, ld), float("nan"), device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_indexer_scores(t["qI"], t["w"], t["kI"], None, 0, 0, 64, 1, N, N, H_I, D_I, None, sc, ld, ds)
    got = sc.cpu().numpy()
    assert status(ds) == 0
    r = np.arange(N) if rows is None else np.unique(np.r_[np.linspace(0, N - 1, rows).astype(int), 0, 127, 128])
    want = oracle.indexer(inp["qI"][r], inp["w"][r], inp["kI"], r)
    for i, t_ in enumerate(r):
        assert np.array_equal(got[t_, :t_ + 1], want[i, :t_ + 1]), t_


def test_indexer_decode_contiguous_and_paged(sa):
    lengths = [131072, 5000, 1, 64, 65, 130000]
    B = len(lengths)
    for paged in (False, True):
        inp = gen_decode(B=B, lengths=lengths, Hq=16, d=64, H_I=8, D_I=64, paged=paged, seed=5)
        t = _to_dev(inp, ("qI", "w", "kI"))
        sl = dev(inp["lengths"])
        if paged:
            S = inp["page_table"].shape[1] * 64
            pt, mp, pp = dev(inp["page_table"]), inp["page_table"].shape[1], inp["kI"].shape[0]
        else:
            S, pt, mp, pp = inp["kI"].shape[1], None, 0, 0
        sc = torch.full((B, S), float("nan"), device="cuda")
        ds = torch.zeros(1, dtype=torch.int32, device="cuda")
        sa.sa_indexer_scores(t["qI"], t["w"], t["kI"], pt, mp, pp, 64, B, 1, S, 8, 64, sl, sc, S, ds)
        got = sc.cpu().numpy()
        assert status(ds) == 0
        for b, L in enumerate(lengths):
            _, _, kI = oracle.decode_sequence(inp, b)
            want = oracle.indexer(inp["qI"][b:b + 1], inp["w"][b:b + 1], kI, [L - 1])
            assert np.array_equal(got[b, :L], want[0]), (paged, b)


# ---------------------------------------------------------------- FP8 indexer
def _e4m3_dev(sa, x_bf16):
    out = torch.empty(x_bf16.shape, dtype=torch.uint8, device="cuda")
    sa.sa_convert_e4m3(x_bf16, out, x_bf16.numel())
    return out


def test_convert_e4m3_matches_oracle(sa):
    r = np.random.default_rng(11)
    vals = (r.standard_normal(300007) * np.exp2(r.uniform(-14, 10, 300007))).astype(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 448, 464, 480, 1e30, -1e30, 2.0 ** -9, 2.0 ** -10,
                        3 * 2.0 ** -10, 2.0 ** -17, 1.0625, 1.1875, -3, 3], dtype=np.float32)
    vals = np.concatenate([special, vals])
    bits = bf16_bits(vals.astype(np.float64))
    x = dev(bits)
    want = oracle.e4m3_encode(bits)
    for lo, n in ((0, bits.size), (0, 1), (0, 7), (0, 9), (1, 1000), (3, 4099)):   # ragged, misaligned
        out = torch.full((n,), 0x55, dtype=torch.uint8, device="cuda")
        sa.sa_convert_e4m3(x[lo:lo + n], out, n)
        assert np.array_equal(out.cpu().numpy(), want[lo:lo + n]), (lo, n)
    nan = dev(bf16_bits(np.array([np.nan, -np.nan])))
    out = _e4m3_dev(sa, nan).cpu().numpy()
    assert np.all(out & 0x7F == 0x7F)


@pytest.mark.parametrize("N,H_I,D_I,rows", [
    (512, 2, 64, None), (1000, 4, 64, None), (300, 8, 128, None), (777, 1, 128, None),
    (129, 4, 64, None), (1, 4, 64, None), (8192, 4, 64, 384), (8192, 8, 128, 200),
    (2, 8, 64, None), (4, 4, 64, None), (3, 4, 64, None),   # 16-column tile: paired rows iff S even
])
def test_indexer_fp8_prefill_exact(sa, N, H_I, D_I, rows):
    inp = gen_prefill(N=N, Hq=1, d=64, H_I=H_I, D_I=D_I, seed=N + 7 * H_I)
    t = _to_dev(inp, ("qI", "w", "kI"))
    q8, k8 = _e4m3_dev(sa, t["qI"]), _e4m3_dev(sa, t["kI"])
    ld = (N + 3) // 4 * 4
    sc = torch.full((N, ld), float("nan"), device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_indexer_scores_fp8(q8, t["w"], k8, None, 0, 0, 64, 1, N, N, H_I, D_I, None, sc, ld, ds)
    got = sc.cpu().numpy()
    assert status(ds) == 0
    r = np.arange(N) if rows is None else np.unique(np.r_[np.linspace(0, N - 1, rows).astype(int), 0, 127, 128])
    qc, kc = oracle.e4m3_encode(inp["qI"][r]), oracle.e4m3_encode(inp["kI"])
    want = oracle.indexer_fp8(qc, inp["w"][r], kc, r)
    for i, t_ in enumerate(r):
        assert np.array_equal(got[t_, :t_ + 1], want[i, :t_ + 1]), t_


def test_indexer_fp8_general_codes_within_fp32_sum_bound(sa):
    # non-integer e4m3 operands: every product is exact, only the fp32 sums
    # round; bound each score by the textbook bound for n fp32 additions,
    # n * 2^-24 of the sum of the terms' magnitudes (n = D_I + H_I)
    N, H_I, D_I = 640, 4, 128
    r = np.random.default_rng(3)
    codes = r.integers(0, 256, size=(N * H_I * D_I + N * D_I,), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38   # no NaN
    qc = codes[:N * H_I * D_I].reshape(N, H_I, D_I)
    kc = codes[N * H_I * D_I:].reshape(N, D_I)
    inp = gen_prefill(N=N, Hq=1, d=64, H_I=H_I, D_I=D_I, seed=4)
    sc = torch.full((N, N), float("nan"), device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_indexer_scores_fp8(dev(qc), dev(inp["w"]), dev(kc), None, 0, 0, 64, 1, N, N, H_I, D_I, None,
                             sc, N, ds)
    got = sc.cpu().numpy()
    assert status(ds) == 0
    rows = np.arange(0, N, 7)
    want = oracle.indexer_fp8(qc[rows], inp["w"][rows], kc, rows)
    qv, kv, wv = oracle.e4m3_decode(qc[rows]), oracle.e4m3_decode(kc), bf16_to_f64(inp["w"][rows])
    mag = np.einsum("rj,rjc,sc->rs", wv, np.abs(qv), np.abs(kv))
    for i, t_ in enumerate(rows):
        err = np.abs(got[t_, :t_ + 1] - want[i, :t_ + 1])
        assert np.all(err <= (D_I + H_I) * 2.0 ** -24 * mag[i, :t_ + 1]), (t_, err.max())


@pytest.mark.parametrize("lengths", [[1, 2, 3, 255, 256, 257, 511, 1000],   # even S: two keys per TMA row
                                     [1, 999, 513, 64]])                     # odd S: one key per row
def test_indexer_fp8_decode_edge_lengths(sa, lengths):
    B = len(lengths)
    for paged in (False, True):
        inp = gen_decode(B=B, lengths=lengths, Hq=16, d=64, H_I=8, D_I=64, paged=paged, seed=8)
        t = _to_dev(inp, ("qI", "w", "kI"))
        q8, k8 = _e4m3_dev(sa, t["qI"]), _e4m3_dev(sa, t["kI"])
        if paged:
            S = inp["page_table"].shape[1] * 64
            pt, mp, pp = dev(inp["page_table"]), inp["page_table"].shape[1], inp["kI"].shape[0]
        else:
            S, pt, mp, pp = inp["kI"].shape[1], None, 0, 0
        ld = (S + 3) // 4 * 4
        sc = torch.full((B, ld), float("nan"), device="cuda")
        ds = torch.zeros(1, dtype=torch.int32, device="cuda")
        sa.sa_indexer_scores_fp8(q8, t["w"], k8, pt, mp, pp, 64, B, 1, S, 8, 64, dev(inp["lengths"]), sc, ld, ds)
        got = sc.cpu().numpy()
        assert status(ds) == 0
        for b, L in enumerate(lengths):
            _, _, kI = oracle.decode_sequence(inp, b)
            want = oracle.indexer_fp8(oracle.e4m3_encode(inp["qI"][b:b + 1]), inp["w"][b:b + 1],
                                      oracle.e4m3_encode(kI), [L - 1])
            assert np.array_equal(got[b, :L], want[0]), (paged, b)
            assert np.all(np.isnan(got[b, L:S])), (paged, b)   # columns past the row are not written


def test_indexer_fp8_decode_contiguous_and_paged(sa):
    lengths = [131072, 5000, 1, 64, 65, 130000]
    B = len(lengths)
    for paged in (False, True):
        inp = gen_decode(B=B, lengths=lengths, Hq=16, d=64, H_I=8, D_I=64, paged=paged, seed=6)
        t = _to_dev(inp, ("qI", "w", "kI"))
        q8, k8 = _e4m3_dev(sa, t["qI"]), _e4m3_dev(sa, t["kI"])
        sl = dev(inp["lengths"])
        if paged:
            S = inp["page_table"].shape[1] * 64
            pt, mp, pp = dev(inp["page_table"]), inp["page_table"].shape[1], inp["kI"].shape[0]
        else:
            S, pt, mp, pp = inp["kI"].shape[1], None, 0, 0
        sc = torch.full((B, S), float("nan"), device="cuda")
        ds = torch.zeros(1, dtype=torch.int32, device="cuda")
        sa.sa_indexer_scores_fp8(q8, t["w"], k8, pt, mp, pp, 64, B, 1, S, 8, 64, sl, sc, S, ds)
        got = sc.cpu().numpy()
        assert status(ds) == 0
        for b, L in enumerate(lengths):
            _, _, kI = oracle.decode_sequence(inp, b)
            want = oracle.indexer_fp8(oracle.e4m3_encode(inp["qI"][b:b + 1]), inp["w"][b:b + 1],
                                      oracle.e4m3_encode(kI), [L - 1])
            assert np.array_equal(got[b, :L], want[0]), (paged, b)


@pytest.mark.parametrize("N,keep,H_I,D_I,rows", [(1000, 4, 4, 64, None), (4096, 16, 8, 64, 200),
                                                   (700, 3, 2, 32, None), (333, 8, 1, 32, None),
                                                   (65, 2, 4, 64, None), (4160, 64, 4, 64, 150)])
def test_block_scores_match_oracle(sa, N, keep, H_I, D_I, rows):
    inp = gen_prefill(N=N, Hq=1, d=64, H_I=H_I, D_I=D_I, seed=N + keep)
    allr = np.arange(N)
    _, blocks = oracle.two_stage(allr, inp["qI"], inp["w"], inp["kI"], 64, keep, 1)   # the oracle's kept blocks
    ld = (keep * 64 + 64 + 3) // 4 * 4
    sc = torch.full((N, ld), float("nan"), device="cuda")
    nbytes = sa.sa_block_scores_workspace_bytes(N, N, keep)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = _to_dev(inp, ("qI", "w", "kI"))
    sa.sa_indexer_scores_blocks(t["qI"], t["w"], t["kI"], N, N, H_I, D_I, dev(blocks.astype(np.int32)), keep, 64,
                                sc, ld, ws, nbytes, ds)
    got = sc.cpu().numpy()
    assert status(ds) == 0
    r = allr if rows is None else np.unique(np.r_[np.linspace(0, N - 1, rows).astype(int), 63, 64, N - 1])
    full = oracle.indexer(inp["qI"][r], inp["w"][r], inp["kI"], r)
    for i, t_ in enumerate(r):
        kept = [b for b in blocks[t_] if b >= 0]
        cand = [b * 64 + j for b in kept for j in range(64)] + list(range((t_ // 64) * 64, t_ + 1))
        assert np.array_equal(got[t_, :len(cand)], full[i, cand]), t_


# ====================================================================== attention
@pytest.mark.parametrize("use_ws", [False, True])
@pytest.mark.parametrize("N,Hq,d,K,W", [
    (512, 4, 64, 64, 32), (700, 16, 128, 100, 17), (300, 20, 64, 50, 0), (257, 64, 128, 64, 64),
    (90, 16, 128, 200, 8), (1, 16, 128, 4, 4), (200, 32, 64, 0, 5), (1000, 8, 128, 300, 40),
    (130, 32, 64, 64, 0), (2048, 16, 128, 256, 64), (1500, 4, 128, 64, 1),
    (3000, 32, 128, 2048, 512), (600, 16, 128, 0, 33), (5000, 16, 128, 2048, 512), (777, 12, 128, 129, 127),
    (400, 16, 128, 2500, 16),
])
def test_prefill_attention_given_oracle_topk(sa, N, Hq, d, K, W, use_ws):
    # use_ws=False: the gathered kernel; True: the masked tensor-core kernel
    # whenever the shape qualifies (sa_prefill_workspace_bytes > 0)
    inp = gen_prefill(N=N, Hq=Hq, d=d, H_I=2, D_I=32, seed=N + Hq)
    t = _to_dev(inp, ("q", "k", "v"))
    if K > 0:
        sc = oracle.indexer(inp["qI"], inp["w"], inp["kI"], np.arange(N))
        top = oracle.topk(sc, np.arange(N) + 1, K)
        top_d = dev(top.astype(np.int32))
    else:
        top, top_d = np.zeros((N, 0), np.int64), None
    out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((N, Hq), dtype=torch.float32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    nb = sa.sa_prefill_workspace_bytes(N, N, K, W, Hq, d) if use_ws else 0
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device="cuda") if nb else None
    sa.sa_sparse_attn_prefill(t["q"], t["k"], t["v"], top_d, K, W, N, N, Hq, d, 1 / math.sqrt(d), out, lse,
                              ws, nb, ds)
    ptr, idx = oracle.selection(top, W, np.arange(N))
    o, l = oracle.sparse_attention(inp["q"], inp["k"], inp["v"], ptr, idx, 1 / math.sqrt(d))
    assert status(ds) == 0
    assert_close_attention(host_f64(out), o, "out")
    assert np.max(np.abs(host_f64(lse) - l)) < 1e-3


def test_prefill_gathered_chunk_two_stage_shape(sa):
    # the last 600 queries of a 70000-token sequence at the two-stage
    # workload's attention shape (16 heads, d=128, K=2048, W=512): more queries
    # than SMs, so the persistent CTAs take several queries each
    S, T, Hq, d, K, W = 70000, 600, 16, 128, 2048, 512
    inp = gen_prefill(N=S, Hq=Hq, d=d, H_I=2, D_I=32, seed=8)
    pos = np.arange(S - T, S)
    sc = oracle.indexer(inp["qI"][S - T:], inp["w"][S - T:], inp["kI"], pos)
    top = oracle.topk(sc, pos + 1, K)
    q = dev(np.ascontiguousarray(inp["q"][S - T:]))
    t = _to_dev(inp, ("k", "v"))
    out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, Hq), dtype=torch.float32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_sparse_attn_prefill(q, t["k"], t["v"], dev(top.astype(np.int32)), K, W, T, S, Hq, d, 1 / math.sqrt(d),
                              out, lse, None, 0, ds)
    ptr, idx = oracle.selection(top, W, pos)
    o, l = oracle.sparse_attention(inp["q"][S - T:], inp["k"], inp["v"], ptr, idx, 1 / math.sqrt(d))
    assert status(ds) == 0
    assert_close_attention(host_f64(out), o, "out")
    assert np.max(np.abs(host_f64(lse) - l)) < 1e-3


@pytest.mark.parametrize("use_ws", [False, True])
def test_prefill_chunk_of_long_sequence(sa, use_ws):
    # the last T queries of an S-token sequence (T < S); with use_ws the masked
    # kernel runs and, at this S, its selection bitmap takes one row per CTA
    S, T, Hq, d, K, W = 100000, 48, 4, 64, 2048, 64
    inp = gen_prefill(N=S, Hq=Hq, d=d, H_I=2, D_I=32, seed=7)
    pos = np.arange(S - T, S)
    sc = oracle.indexer(inp["qI"][S - T:], inp["w"][S - T:], inp["kI"], pos)
    top = oracle.topk(sc, pos + 1, K)
    q = dev(np.ascontiguousarray(inp["q"][S - T:]))
    t = _to_dev(inp, ("k", "v"))
    out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, Hq), dtype=torch.float32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    nb = sa.sa_prefill_workspace_bytes(T, S, K, W, Hq, d) if use_ws else 0
    if use_ws:
        assert nb > 0   # the shape qualifies for the masked kernel
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda") if nb else None
    sa.sa_sparse_attn_prefill(q, t["k"], t["v"], dev(top.astype(np.int32)), K, W, T, S, Hq, d, 1 / math.sqrt(d),
                              out, lse, ws, nb, ds)
    ptr, idx = oracle.selection(top, W, pos)
    o, l = oracle.sparse_attention(inp["q"][S - T:], inp["k"], inp["v"], ptr, idx, 1 / math.sqrt(d))
    assert status(ds) == 0
    assert_close_attention(host_f64(out), o, "out")
    assert np.max(np.abs(host_f64(lse) - l)) < 1e-3


# ====================================================================== end to end
def _prefill_e2e(sa, inp, K, W, rows=None, block=None, keep=None, index_fp8=False):
    PrefillPlan, _ = _pl()
    N, Hq, d = inp["q"].shape
    H_I, D_I = inp["qI"].shape[1:]
    plan = PrefillPlan(N, Hq, d, H_I, D_I, K, W, block=block, keep=keep, index_fp8=index_fp8)
    t = _to_dev(inp)
    if index_fp8:   # the integer indexer inputs are exact in e4m3: same oracle
        t["qI"], t["kI"] = _e4m3_dev(sa, t["qI"]), _e4m3_dev(sa, t["kI"])
    plan.run(t["q"], t["k"], t["v"], t["qI"], t["w"], t["kI"])
    assert status(plan.dev_status) == 0
    ref = oracle.prefill(inp, K, W, rows=rows, block=block, keep=keep)
    r = np.arange(N) if rows is None else np.asarray(rows)
    assert np.array_equal(plan.topk.cpu().numpy()[r], ref["topk"])
    assert_close_attention(host_f64(plan.out)[r], ref["out"], "out")
    assert np.max(np.abs(host_f64(plan.lse)[r] - ref["lse"])) < 1e-3
    return plan, ref


@pytest.mark.parametrize("T,S,block,keep,K,W", [(300, 5000, None, None, 512, 64), (700, 4096, 64, 16, 512, 64)])
def test_plan_for_the_last_rows_of_a_longer_sequence(sa, T, S, block, keep, K, W):
    # one rank's share of a query-row partition: T queries at positions
    # S - T .. S - 1 over S keys, against the oracle on those rows
    PrefillPlan, _ = _pl()
    inp = gen_prefill(N=S, Hq=16, d=128, H_I=4, D_I=64, seed=T + S)
    plan = PrefillPlan(T, 16, 128, 4, 64, K, W, block=block, keep=keep, S=S)
    q, qI, w = (dev(np.ascontiguousarray(inp[n][S - T:])) for n in ("q", "qI", "w"))
    t = _to_dev(inp, ("k", "v", "kI"))
    plan.run(q, t["k"], t["v"], qI, w, t["kI"])
    assert status(plan.dev_status) == 0
    ref = oracle.prefill(inp, K, W, rows=np.arange(S - T, S), block=block, keep=keep)
    assert np.array_equal(plan.topk.cpu().numpy(), ref["topk"])
    assert_close_attention(host_f64(plan.out), ref["out"], "out")
    assert np.max(np.abs(host_f64(plan.lse) - ref["lse"])) < 1e-3


def test_host_pipeline_matches_direct_runs(sa):
    # three steps with different inputs through the overlapped host-buffer
    # runner: each downloaded output equals a direct run of the plan
    from fine_grained_top_b200.pipeline import HostPipeline
    PrefillPlan, _ = _pl()
    c = CONFIGS["prefill_512"]
    names = ("q", "k", "v", "qI", "w", "kI")
    steps = [gen_prefill(seed=s, **c) for s in (0, 1, 2)]
    hin = [{n: dev(st[n]).cpu().pin_memory() for n in names} for st in steps]
    make = lambda: PrefillPlan(c["N"], c["Hq"], c["d"], c["H_I"], c["D_I"], c["K"], c["W"])
    pipe = HostPipeline(make, hin[0])
    outs = [torch.empty((c["N"], c["Hq"], c["d"]), dtype=torch.bfloat16).pin_memory() for _ in steps]
    pipe.run(hin, outs)
    torch.cuda.synchronize()
    assert pipe.dev_status() == 0
    for st, o in zip(steps, outs):
        plan = make()
        t = _to_dev(st)
        plan.run(t["q"], t["k"], t["v"], t["qI"], t["w"], t["kI"])
        assert torch.equal(o, plan.out.cpu())
    assert not torch.equal(outs[0], outs[1])


def test_row_blocked_scoring_matches_whole(sa):
    # scoring and selecting in row blocks gives the same step as one launch each
    PrefillPlan, _ = _pl()
    c = CONFIGS["prefill_512"]
    inp = config_inputs("prefill_512")
    t = _to_dev(inp)
    plans = [PrefillPlan(c["N"], c["Hq"], c["d"], c["H_I"], c["D_I"], c["K"], c["W"], row_blocks=rb)
             for rb in (1, 3)]
    for p in plans:
        p.run(t["q"], t["k"], t["v"], t["qI"], t["w"], t["kI"])
        assert status(p.dev_status) == 0
    assert torch.equal(plans[0].topk, plans[1].topk)
    assert torch.equal(plans[0].out, plans[1].out)
    assert plans[1].launches() == 2 * 3 + 1


def test_e2e_prefill_512(sa):
    c = CONFIGS["prefill_512"]
    _prefill_e2e(sa, config_inputs("prefill_512"), c["K"], c["W"])


@pytest.mark.parametrize("index_fp8", [False, True])
def test_e2e_prefill_8k(sa, index_fp8):
    c = CONFIGS["prefill_8k"]
    inp = config_inputs("prefill_8k")
    N = c["N"]
    rows = np.unique(np.r_[np.linspace(0, N - 1, 160).astype(int), 1023, 1024, 1151, 1152, N - 1])
    plan, _ = _prefill_e2e(sa, inp, c["K"], c["W"], rows=rows, index_fp8=index_fp8)
    # every row's index set, bit for bit (the oracle's selection of all 8192 rows)
    sc = oracle.indexer(inp["qI"], inp["w"], inp["kI"], np.arange(N))
    want = oracle.topk(sc, np.arange(N) + 1, c["K"])
    assert np.array_equal(plan.topk.cpu().numpy(), want)


@pytest.mark.parametrize("N,block,keep,K,W", [(1000, 64, 4, 100, 16), (4096, 64, 16, 512, 64),
                                               (640, 64, 100, 300, 8)])
def test_e2e_two_stage_small(sa, N, block, keep, K, W):
    inp = gen_prefill(N=N, Hq=16, d=128, H_I=4, D_I=64, seed=N + keep)
    _prefill_e2e(sa, inp, K, W, block=block, keep=keep)


def test_e2e_two_stage_64k(sa):
    # every row's kept blocks and fine top-K index set, bit for bit; attention
    # outputs on 2100+ rows: evenly spaced ones plus block, window and
    # selection-size edges
    c = CONFIGS["prefill_64k_two_stage"]
    inp = config_inputs("prefill_64k_two_stage")
    N, blk, keep, K, W = c["N"], c["block"], c["keep"], c["K"], c["W"]
    edges = []
    for e in (63, 64, 65, 511, 512, 513, 2047, 2048, 2559, 2560, 2561, 4095, 4096, 4159, 4160, 4161, 4223,
              4224, 32767, 32768, N - 65, N - 64, N - 2, N - 1):
        edges += [e - 1, e, e + 1]
    rows = np.unique(np.clip(np.r_[np.linspace(0, N - 1, 2048).astype(int), edges], 0, N - 1))
    plan, ref = _prefill_e2e(sa, inp, K, W, rows=rows, block=blk, keep=keep)
    assert len(rows) >= 2048
    assert np.array_equal(plan.blocks.cpu().numpy()[rows], ref["blocks"])
    all_rows = np.arange(N, dtype=np.int64)
    want_top, want_blocks = oracle.two_stage(all_rows, inp["qI"], inp["w"], inp["kI"], blk, keep, K)
    assert np.array_equal(plan.blocks.cpu().numpy(), want_blocks)
    assert np.array_equal(plan.topk.cpu().numpy(), want_top)


def _decode_e2e(sa, inp, K, W, index_fp8=False, fused=None):
    _, DecodePlan = _pl()
    B, Hq, d = inp["q"].shape
    H_I, D_I = inp["qI"].shape[1:]
    paged = "page_table" in inp
    t = _to_dev(inp)
    if index_fp8:   # the integer indexer inputs are exact in e4m3: same oracle
        t["qI"], t["kI"] = _e4m3_dev(sa, t["qI"]), _e4m3_dev(sa, t["kI"])
    sl = dev(inp["lengths"])
    if paged:
        pt = dev(inp["page_table"])
        plan = DecodePlan(B, Hq, d, H_I, D_I, K, W, S_max=0, paged=True,
                          max_pages=inp["page_table"].shape[1], pool_pages=inp["k"].shape[0],
                          index_fp8=index_fp8, fused=fused)
    else:
        pt = None
        plan = DecodePlan(B, Hq, d, H_I, D_I, K, W, S_max=inp["k"].shape[1], index_fp8=index_fp8, fused=fused)
    plan.run(t["q"], t["k"], t["v"], t["qI"], t["w"], t["kI"], sl, pt)
    assert status(plan.dev_status) == 0
    ref = oracle.decode(inp, K, W)
    assert np.array_equal(plan.topk.cpu().numpy(), ref["topk"])
    assert_close_attention(host_f64(plan.out), ref["out"], "decode out")
    assert np.max(np.abs(host_f64(plan.lse) - ref["lse"])) < 1e-3


# (bf16 indexer fused with the top-K, the same two kernels apart, the FP8 indexer)
DECODE_SELECTIONS = [(False, True), (False, False), (True, False)]


@pytest.mark.parametrize("index_fp8,fused", DECODE_SELECTIONS)
def test_e2e_decode_8x128k(sa, index_fp8, fused):
    c = CONFIGS["decode_8x128k"]
    _decode_e2e(sa, config_inputs("decode_8x128k"), c["K"], c["W"], index_fp8=index_fp8, fused=fused)


@pytest.mark.parametrize("index_fp8,fused", DECODE_SELECTIONS)
def test_e2e_decode_paged_16(sa, index_fp8, fused):
    c = CONFIGS["decode_paged_16x256k"]
    _decode_e2e(sa, config_inputs("decode_paged_16x256k"), c["K"], c["W"], index_fp8=index_fp8, fused=fused)


@pytest.mark.parametrize("paged", [False, True])
@pytest.mark.parametrize("H_I,D_I", [(8, 64), (4, 128), (3, 64), (1, 128)])
def test_fused_indexer_topk_decode_matches_oracle(sa, paged, H_I, D_I):
    # lengths around the 256-key tiles, the 8192-key chunks of a cluster CTA
    # and K; one sequence of a single key; heads below 8 leave MMA columns empty
    lengths = [131072, 5000, 1, 2048, 2049, 8193, 255, 70001]
    B, K = len(lengths), 2048
    inp = gen_decode(B=B, lengths=lengths, Hq=8, d=64, H_I=H_I, D_I=D_I, paged=paged, seed=6)
    t = _to_dev(inp, ("qI", "w", "kI"))
    sl = dev(inp["lengths"])
    if paged:
        S = inp["page_table"].shape[1] * 64
        pt, mp, pp = dev(inp["page_table"]), inp["page_table"].shape[1], inp["kI"].shape[0]
    else:
        S, pt, mp, pp = inp["kI"].shape[1], None, 0, 0
    topk = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_indexer_topk_decode(t["qI"], t["w"], t["kI"], pt, mp, pp, 64, B, S, H_I, D_I, sl, K, topk, ds)
    got = topk.cpu().numpy()
    assert status(ds) == 0
    for b, L in enumerate(lengths):
        _, _, kI = oracle.decode_sequence(inp, b)
        sc = oracle.indexer(inp["qI"][b:b + 1], inp["w"][b:b + 1], kI, [L - 1])
        want = oracle.topk(sc, [L], K)
        assert np.array_equal(got[b], want[0]), (paged, b)


@pytest.mark.parametrize("lengths,K,W", [([1, 2, 63, 64, 65, 3000], 100, 16), ([5000, 700], 4096, 0),
                                         ([129, 10000], 0, 600)])
def test_decode_edge_lengths(sa, lengths, K, W):
    for paged in (False, True):
        inp = gen_decode(B=len(lengths), lengths=lengths, Hq=64, d=128, H_I=8, D_I=64, paged=paged, seed=11)
        _decode_e2e(sa, inp, K, W)


@pytest.mark.parametrize("paged", [False, True])
def test_decode_split_k_merge_matches_oracle(sa, paged):
    # K + W > 16 * 1024 leaves more than 1024 keys per CTA of a 16-CTA cluster,
    # so sa_sparse_attn_decode takes its split-K path: partial states in the
    # caller's workspace, merged by decode_merge_kernel
    K, W = 16000, 1000
    lengths = [40000, 17001, 16999, 5000, 90000, 1]
    inp = gen_decode(B=len(lengths), lengths=lengths, Hq=64, d=128, H_I=8, D_I=64, paged=paged, seed=31)
    _, DecodePlan = _pl()
    B = len(lengths)
    if paged:
        plan = DecodePlan(B, 64, 128, 8, 64, K, W, S_max=0, paged=True, max_pages=inp["page_table"].shape[1],
                          pool_pages=inp["k"].shape[0])
    else:
        plan = DecodePlan(B, 64, 128, 8, 64, K, W, S_max=inp["k"].shape[1])
    assert plan.launches() == 4   # indexer, top-K, split-K attention, merge
    _decode_e2e(sa, inp, K, W)


# ====================================================================== device errors
@pytest.mark.parametrize("use_ws", [False, True])
def test_planted_bad_index_and_order_are_reported(sa, use_ws):
    N, Hq, d, K, W = 100, 16, 128, 8, 4
    inp = gen_prefill(N=N, Hq=Hq, d=d, H_I=2, D_I=32, seed=1)
    t = _to_dev(inp, ("q", "k", "v"))
    nb = sa.sa_prefill_workspace_bytes(N, N, K, W, Hq, d) if use_ws else 0
    assert nb > 0 or not use_ws
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device="cuda") if nb else None
    top = np.tile(np.arange(K, dtype=np.int32), (N, 1))
    top[50, 3] = 99            # beyond position 50
    out = torch.empty((N, Hq, d), dtype=torch.bfloat16, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_sparse_attn_prefill(t["q"], t["k"], t["v"], dev(top), K, W, N, N, Hq, d, 0.1, out, None, ws, nb, ds)
    assert status(ds) & sa.SA_DEV_INDEX
    assert torch.isfinite(out.float()).all()
    top2 = np.tile(np.arange(K, dtype=np.int32), (N, 1))
    top2[60, 2], top2[60, 3] = 5, 4   # not ascending
    ds.zero_()
    sa.sa_sparse_attn_prefill(t["q"], t["k"], t["v"], dev(top2), K, W, N, N, Hq, d, 0.1, out, None, ws, nb, ds)
    assert status(ds) & sa.SA_DEV_ORDER


def test_planted_bad_page_is_reported(sa):
    inp = gen_decode(B=2, lengths=[300, 200], Hq=16, d=128, H_I=8, D_I=64, paged=True, seed=2)
    inp["page_table"][1, 1] = 10 ** 6
    _, DecodePlan = _pl()
    t = _to_dev(inp)
    plan = DecodePlan(2, 16, 128, 8, 64, 16, 8, S_max=0, paged=True, max_pages=inp["page_table"].shape[1],
                      pool_pages=inp["k"].shape[0])
    plan.run(t["q"], t["k"], t["v"], t["qI"], t["w"], t["kI"], dev(inp["lengths"]), dev(inp["page_table"]))
    assert status(plan.dev_status) & sa.SA_DEV_INDEX
    assert torch.isfinite(plan.out.float()).all()


def test_fused_select_reports_bad_page_and_length(sa):
    # a page id outside the pool among the pages of a scored sequence, and a
    # sequence length beyond S, are reported; the other rows' selections stand
    inp = gen_decode(B=3, lengths=[3000, 2500, 4000], Hq=8, d=64, H_I=8, D_I=64, paged=True, seed=12)
    table = inp["page_table"].copy()
    table[1, 5] = 10 ** 6
    S = table.shape[1] * 64
    lengths = inp["lengths"].copy()
    t = _to_dev(inp, ("qI", "w", "kI"))
    K = 1024
    topk = torch.empty((3, K), dtype=torch.int32, device="cuda")
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_indexer_topk_decode(t["qI"], t["w"], t["kI"], dev(table), table.shape[1], inp["kI"].shape[0], 64, 3, S,
                              8, 64, dev(lengths), K, topk, ds)
    assert status(ds) & sa.SA_DEV_INDEX
    got = topk.cpu().numpy()
    for b in (0, 2):
        _, _, kI = oracle.decode_sequence(inp, b)
        want = oracle.topk(oracle.indexer(inp["qI"][b:b + 1], inp["w"][b:b + 1], kI, [lengths[b] - 1]),
                           [lengths[b]], K)
        assert np.array_equal(got[b], want[0]), b
    lengths[2] = S + 1   # longer than the row
    ds.zero_()
    sa.sa_indexer_topk_decode(t["qI"], t["w"], t["kI"], dev(inp["page_table"]), table.shape[1], inp["kI"].shape[0],
                              64, 3, S, 8, 64, dev(lengths), K, topk, ds)
    assert status(ds) & sa.SA_DEV_INDEX


def test_bounded_wait_reports_timeout_and_context_survives(sa):
    # a wait on a barrier that nothing arrives at gives up after 20 ms and
    # reports SA_DEV_TIMEOUT; the context keeps working afterwards
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_selftest_wait_timeout(20000, ds)
    assert status(ds) == sa.SA_DEV_TIMEOUT
    assert sa.sa_dev_status_decode(status(ds)) == sa.SA_ERR_TIMEOUT
    sc = torch.arange(64, dtype=torch.float32, device="cuda").reshape(1, 64)
    out = torch.empty((1, 4), dtype=torch.int32, device="cuda")
    sa.sa_topk_select(sc, 64, 1, 64, None, None, 0, 4, out)
    assert out.cpu().tolist() == [[60, 61, 62, 63]]
