"""Pins for the CPU oracle: each test ties it to something other than itself.

Closed forms, brute force on tiny inputs, identities of the definitions and
the pages' own formulas.  A plausible mistake in the oracle (a dropped ReLU or
weight, a wrong sign or index, an off-by-one window, a wrong tie rule, a
missing softmax normaliser) fails at least one of these.
"""

import itertools
import math

import numpy as np
import pytest

import oracle
from workloads import bf16_bits, gen_prefill, gen_decode
from tests.conftest import golden_path

rng = np.random.default_rng(12345)


def _sections(path):
    sec, out = None, {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line[0].isalpha():
            sec = line
            out[sec] = []
            continue
        out[sec].append([float(x) for x in line.split()])
    return out


# ---------------------------------------------------------------- indexer
def test_indexer_worked_example():
    g = _sections(golden_path("indexer_worked_example.txt"))
    kI = np.array(g["kI"])
    qI = np.array([g["qI t=1"], g["qI t=2"]])
    w = np.array([g["w t=1"][0], g["w t=2"][0]])
    sc = oracle.indexer(qI, w, kI, lim=[1, 2])
    want = np.array([g["scores t=1"][0], g["scores t=2"][0]])
    assert np.array_equal(sc, want)
    assert np.array_equal(oracle.topk(sc, [2, 3], 1), np.array(g["topk1"], dtype=np.int64))
    assert np.array_equal(oracle.topk(sc, [2, 3], 2), np.array(g["topk2"], dtype=np.int64))


def _rand_index_inputs(R, S, H, D):
    qI = rng.integers(-3, 4, size=(R, H, D)).astype(np.float64)
    w = rng.integers(0, 4, size=(R, H)).astype(np.float64)
    kI = rng.integers(-3, 4, size=(S, D)).astype(np.float64)
    lim = rng.integers(-1, S, size=R)
    return qI, w, kI, lim


def test_indexer_zero_weights_and_zero_keys():
    qI, w, kI, lim = _rand_index_inputs(7, 40, 3, 8)
    causal = np.arange(40)[None, :] <= lim[:, None]
    for sc in (oracle.indexer(qI, np.zeros_like(w), kI, lim),
               oracle.indexer(qI, w, np.zeros_like(kI), lim)):
        assert np.all(sc[causal] == 0.0)
        assert np.all(np.isneginf(sc[~causal]))


def test_indexer_relu_sign_identity():
    # ReLU(x) - ReLU(-x) = x, so I(qI) - I(-qI) = sum_j w_j (qI_j . kI_s):
    # a linear form, catches a dropped / wrong ReLU and a misplaced weight.
    qI, w, kI, lim = _rand_index_inputs(9, 33, 4, 16)
    lim[:] = 32
    diff = oracle.indexer(qI, w, kI, lim) - oracle.indexer(-qI, w, kI, lim)
    lin = np.einsum("rh,rhd,sd->rs", w, qI, kI)
    assert np.array_equal(diff, lin)


def test_indexer_linear_in_w_and_homogeneous_in_kI():
    qI, w, kI, lim = _rand_index_inputs(6, 25, 2, 32)
    w2 = rng.integers(0, 4, size=w.shape).astype(np.float64)
    a = oracle.indexer(qI, w, kI, lim)
    b = oracle.indexer(qI, w2, kI, lim)
    ab = oracle.indexer(qI, w + w2, kI, lim)
    fin = np.isfinite(ab)
    assert np.array_equal(ab[fin], (a + b)[fin])
    assert np.array_equal(oracle.indexer(qI, w, 2.0 * kI, lim)[fin], 2.0 * a[fin])


def test_indexer_one_hot_closed_form():
    # qI[t,j] = alpha_j e_a, kI[s] = beta_s e_{b_s}:
    # I = sum_j w_j max(0, alpha_j beta_s) when b_s == a, else 0.
    D, H, S = 8, 3, 12
    alpha = np.array([2.0, -1.0, 3.0])
    w = np.array([[1.0, 2.0, 3.0]])
    qI = np.zeros((1, H, D)); qI[0, :, 5] = alpha
    kI = np.zeros((S, D))
    beta = np.array([1, -2, 3, 0, -1, 2, 1, 1, -3, 2, 2, 1], dtype=np.float64)
    pos = np.array([5, 5, 5, 5, 5, 1, 2, 5, 5, 0, 5, 7])
    kI[np.arange(S), pos] = beta
    sc = oracle.indexer(qI, w, kI, [S - 1])[0]
    for s in range(S):
        want = sum(w[0, j] * max(0.0, alpha[j] * beta[s]) for j in range(H)) if pos[s] == 5 else 0.0
        assert sc[s] == want


def test_indexer_exact_integer_bound_on_workload_inputs():
    inp = gen_prefill(N=300, Hq=2, d=64, H_I=8, D_I=64, seed=3)
    sc = oracle.indexer(inp["qI"], inp["w"], inp["kI"], np.arange(300))
    fin = sc[np.isfinite(sc)]
    assert np.array_equal(fin, np.round(fin))
    assert fin.min() >= 0 and fin.max() <= 8 * 3 * 64 * 9
    assert np.all(np.isneginf(sc[np.triu_indices(300, 1)]))


# ---------------------------------------------------------------- e4m3 operands
# The FP8 indexer reading: OCP e4m3, round to nearest even, +-448 saturation.
def test_e4m3_decode_matches_torch_on_every_code():
    torch = pytest.importorskip("torch")
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    assert np.array_equal(np.nonzero(np.isnan(ours))[0], [0x7F, 0xFF])
    ok = ~np.isnan(ours)
    assert np.array_equal(ours[ok], lib[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(lib[ok]))   # 0x80 is -0


def test_e4m3_encode_matches_torch_inside_the_range():
    torch = pytest.importorskip("torch")
    r = np.random.default_rng(7)
    # float32 values (so torch sees the same number), spread over every binade
    # and the subnormals; |x| < 448, where torch's conversion does not saturate
    x = (r.standard_normal(200000) * np.exp2(r.uniform(-12, 9, 200000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    grid = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    grid = grid[np.isfinite(grid)]
    mids = ((np.sort(grid)[1:] + np.sort(grid)[:-1]) / 2).astype(np.float32)   # every tie, exact in f32
    x = np.concatenate([x, mids[np.abs(mids) < 448]])
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(x.astype(np.float64)), lib)


def test_e4m3_round_trip_ties_and_saturation():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)
    cases = {1.0: 0x38, 1.0625: 0x38, 1.1875: 0x3A, 2.0 ** -9: 0x01, 2.0 ** -10: 0x00,
             3 * 2.0 ** -10: 0x02, 2.0 ** -6: 0x08, 15 * 2.0 ** -10: 0x08, 448.0: 0x7E,
             460.0: 0x7E, 470.0: 0x7E, 480.0: 0x7E, 1e9: 0x7E, -1e9: 0xFE, -math.inf: 0xFE, math.inf: 0x7E, -2.0: 0xC0,
             3.0: 0x44, -3.0: 0xC4, 0.0: 0x00}
    got = oracle.e4m3_encode(np.array(list(cases)))
    assert got.tolist() == list(cases.values())
    assert oracle.e4m3_encode(np.array([math.nan]))[0] == 0x7F


def test_indexer_fp8_equals_indexer_on_small_integers():
    # the integers -3..3 (the indexer inputs of the workloads) are exact in e4m3
    q = rng.integers(-3, 4, size=(6, 2, 32)).astype(np.float64)
    k = rng.integers(-3, 4, size=(40, 32)).astype(np.float64)
    w = rng.integers(0, 4, size=(6, 2)).astype(np.float64)
    lim = np.arange(34, 40)
    a = oracle.indexer(q, w, k, lim)
    b = oracle.indexer_fp8(oracle.e4m3_encode(q), w, oracle.e4m3_encode(k), lim)
    assert np.array_equal(a, b)
    # and a value e4m3 cannot hold moves the score: the codes are really used
    k2 = k.copy()
    k2[0, 0] = 1.1
    b2 = oracle.indexer_fp8(oracle.e4m3_encode(q), w, oracle.e4m3_encode(k2), lim)
    assert np.all(b2[:, 1:] == a[:, 1:])
    assert np.allclose(b2[:, 0], oracle.indexer(q, w, np.where(k2 == 1.1, 1.125, k2), lim)[:, 0])


# ---------------------------------------------------------------- top-K
def _dominates(score, i, j):
    """i ranks strictly above j: higher score, or equal score and lower position."""
    return score[i] > score[j] or (score[i] == score[j] and i < j)


def test_topk_brute_force_all_subsets():
    # The pages' rule (top-K, ties -> lower position) characterised without
    # sorting: the chosen set is the unique subset whose every member ranks
    # above every non-member.
    for trial in range(300):
        L = int(rng.integers(1, 9))
        K = int(rng.integers(0, 5))
        score = rng.integers(0, 3, size=L).astype(np.float64)
        m = min(K, L)
        ok = [c for c in itertools.combinations(range(L), m)
              if all(_dominates(score, i, j) for i in c for j in range(L) if j not in c)]
        assert len(ok) == 1
        got = oracle.topk(score[None, :], [L], K)[0]
        assert list(got[:m]) == list(ok[0]) and np.all(got[m:] == -1)


def test_topk_heavy_ties_property_on_long_rows():
    R, L, K = 5, 3000, 700
    scores = rng.integers(0, 3, size=(R, L)).astype(np.float64)
    n_valid = np.array([3000, 2999, 1500, 700, 10])
    got = oracle.topk(scores, n_valid, K)
    for r in range(R):
        n = n_valid[r]
        m = min(K, n)
        sel = got[r, :m]
        assert np.all(got[r, m:] == -1)
        assert np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < n
        mask = np.zeros(n, bool); mask[sel] = True
        s = scores[r, :n]
        if m < n:
            # worst selected vs best unselected, in the (score desc, pos asc) order
            worst = min(sel, key=lambda i: (s[i], -i))
            uns = np.flatnonzero(~mask)
            best = max(uns, key=lambda i: (s[i], -i))
            assert _dominates(s, worst, best)


def test_topk_degenerate_K():
    scores = rng.standard_normal((3, 50))
    assert np.all(oracle.topk(scores, [50, 20, 0], 0) == np.zeros((3, 0)))
    full = oracle.topk(scores, [50, 20, 0], 60)
    assert list(full[0, :50]) == list(range(50)) and np.all(full[0, 50:] == -1)
    assert list(full[1, :20]) == list(range(20)) and np.all(full[1, 20:] == -1)
    assert np.all(full[2] == -1)


def test_topk_candidate_map():
    score = np.array([[1.0, 5.0, 5.0, 0.0, 7.0]])
    cand = np.array([[3, 10, 11, 40, 41]])
    assert list(oracle.topk(score, [5], 3, cand=cand)[0]) == [10, 11, 41]


# ---------------------------------------------------------------- coarse pass
def test_pool_mean_closed_forms():
    blk, D = 4, 3
    kI = np.zeros((4 * blk + 3, D))
    for b in range(4):
        kI[b * blk:(b + 1) * blk] = [b, -b, 2 * b]      # constant blocks
    kI[4 * blk:] = 99.0                                  # partial tail: dropped
    kB = oracle.pool_mean(kI, blk)
    assert kB.shape == (4, D)
    assert np.array_equal(kB, np.array([[b, -b, 2 * b] for b in range(4)], float))
    ramp = np.arange(64, dtype=np.float64)[:, None] * np.ones((1, 2))
    assert np.array_equal(oracle.pool_mean(ramp, 64), np.full((1, 2), 31.5))


def test_two_stage_keep_all_blocks_equals_single_stage():
    N, blk = 640, 64
    inp = gen_prefill(N=N, Hq=1, d=64, H_I=4, D_I=64, seed=11)
    rows = np.arange(N)
    single = oracle.indexer(inp["qI"], inp["w"], inp["kI"], rows)
    for K in (1, 33, 200, 700):
        want = oracle.topk(single, rows + 1, K)
        got, blocks = oracle.two_stage(rows, inp["qI"], inp["w"], inp["kI"], blk, N // blk, K)
        assert np.array_equal(got, want)
        for t in (0, 63, 64, 127, 639):
            nb = t // blk
            assert list(blocks[t, :nb]) == list(range(nb)) and np.all(blocks[t, nb:] == -1)


def test_two_stage_planted_block_and_own_block():
    # keep = 1: the block whose pooled key matches the query best is kept; the
    # candidates are that block's tokens plus the query's own block up to t.
    blk, N, D = 8, 64, 4
    kI = np.zeros((N, D))
    kI[24:32, 0] = 1.0                      # block 3 points along +e0
    kI[40:48, 0] = -1.0                     # block 5 opposes it
    qI = np.zeros((1, 1, D)); qI[0, 0, 0] = 1.0
    w = np.ones((1, 1))
    t = 53
    top, blocks = oracle.two_stage([t], qI, w, kI, blk, 1, 100)
    assert list(blocks[0]) == [3]
    cand = list(range(24, 32)) + list(range(48, 54))
    assert list(top[0, :len(cand)]) == cand and np.all(top[0, len(cand):] == -1)
    top2, _ = oracle.two_stage([t], qI, w, kI, blk, 1, 8)
    assert list(top2[0]) == list(range(24, 32))      # score 1 beats the own block's 0


def _page_selection_brute(t, qI, w, kI, blk, keep):
    """Plain-Python page selection: pooled block keys, coarse scores, the best
    `keep` eligible blocks (ties to the lower block), their tokens and the
    query's own block up to t, ascending."""
    own = t // blk
    scored = []
    for b in range(own):
        kb = kI[b * blk:(b + 1) * blk].mean(axis=0)
        sc = sum(w[j] * max(0.0, float(np.dot(qI[j], kb))) for j in range(qI.shape[0]))
        scored.append((-sc, b))
    kept = sorted(b for _, b in sorted(scored)[:keep])
    return [s for b in kept for s in range(b * blk, (b + 1) * blk)] + list(range(own * blk, t + 1))


@pytest.mark.parametrize("keep", [0, 1, 3, 50])
def test_page_selection_brute_force(keep):
    blk, N = 8, 160
    inp = gen_prefill(N=N, Hq=1, d=64, H_I=2, D_I=32, seed=21 + keep)   # small integers: many ties
    qI, w, kI = (oracle._f64(inp[x]) for x in ("qI", "w", "kI"))
    rows = np.arange(N)
    pos, blocks = oracle.page_selection(rows, qI, w, kI, blk, keep)
    assert pos.shape == (N, keep * blk + blk)
    for t in rows:
        want = _page_selection_brute(int(t), qI[t], w[t], kI, blk, keep)
        assert list(pos[t, :len(want)]) == want, t
        assert np.all(pos[t, len(want):] == -1), t


def test_page_selection_keeping_every_block_is_dense_causal():
    blk, N = 16, 96
    inp = gen_prefill(N=N, Hq=2, d=64, H_I=2, D_I=32, seed=9)
    keep = N // blk
    res = oracle.prefill(inp, K=keep * blk + blk, W=4, block=blk, keep=keep)
    q, k, v = (oracle._f64(inp[x]) for x in "qkv")
    assert np.max(np.abs(res["out"] - _dense_causal_textbook(q, k, v, 1.0 / 8.0))) < 1e-12


# ---------------------------------------------------------------- selection
def test_selection_window_and_union():
    ptr, idx = oracle.selection(np.array([[-1, -1]]), 3, [0])
    assert list(idx) == [0]
    ptr, idx = oracle.selection(np.array([[2, 7, 9, -1]]), 3, [9])
    assert list(idx) == [2, 7, 8, 9]
    ptr, idx = oracle.selection(np.array([[0, 1], [5, 6]]), 0, [4, 6])
    assert list(idx[ptr[0]:ptr[1]]) == [0, 1] and list(idx[ptr[1]:ptr[2]]) == [5, 6]
    ptr, idx = oracle.selection(np.zeros((1, 0), dtype=np.int64), 4, [2])
    assert list(idx) == [0, 1, 2]


def test_window_matches_golden_mask():
    mask = np.loadtxt(golden_path("window_mask_n6_w3.txt"))
    empty = -np.ones((6, 0), dtype=np.int64)
    ptr, idx = oracle.selection(empty, 3, np.arange(6))
    got = np.zeros((6, 6))
    for i in range(6):
        got[i, idx[ptr[i]:ptr[i + 1]]] = 1
    assert np.array_equal(got, mask)


# ---------------------------------------------------------------- attention
def _dense_causal_textbook(q, k, v, scale):
    """softmax(QK^T/sqrt(d) + causal -inf) V, one full score matrix per head
    ("A Guide to Sparse Attention in Large Models", section 2)."""
    N = q.shape[0]
    out = np.empty_like(q)
    tri = np.triu(np.ones((N, N), bool), 1)
    for h in range(q.shape[1]):
        s = q[:, h, :] @ k.T * scale
        s[tri] = -np.inf
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v
    return out


def _masked_formula(q, k, v, mask, scale):
    """softmax(QK^T * Mask + (1 - Mask)(-inf)) V, literally (same page)."""
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        s = q[:, h, :] @ k.T * scale
        with np.errstate(invalid="ignore"):
            masked = np.where(mask == 1, s * mask, -np.inf)
        p = np.exp(masked - masked.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v
    return out


@pytest.mark.parametrize("N,K,W", [(96, 96, 8), (96, 200, 0), (130, 130, 1)])
def test_attention_K_ge_N_is_dense_causal(N, K, W):
    inp = gen_prefill(N=N, Hq=3, d=64, H_I=2, D_I=32, seed=5)
    res = oracle.prefill(inp, K=K, W=W)
    q, k, v = (oracle._f64(inp[x]) for x in "qkv")
    want = _dense_causal_textbook(q, k, v, 1.0 / 8.0)
    assert np.max(np.abs(res["out"] - want)) < 1e-12


@pytest.mark.parametrize("W", [1, 3, 17])
def test_attention_K0_is_the_masked_window_formula(W):
    N = 64
    inp = gen_prefill(N=N, Hq=2, d=64, H_I=2, D_I=32, seed=6)
    res = oracle.prefill(inp, K=0, W=W)
    i = np.arange(N)[:, None]; j = np.arange(N)[None, :]
    mask = ((i - j >= 0) & (i - j < W)).astype(np.float64)
    q, k, v = (oracle._f64(inp[x]) for x in "qkv")
    want = _masked_formula(q, k, v, mask, 1.0 / 8.0)
    assert np.max(np.abs(res["out"] - want)) < 1e-12


def test_attention_weights_sum_to_one_and_uniform_lse():
    N = 80
    inp = gen_prefill(N=N, Hq=2, d=64, H_I=2, D_I=32, seed=7)
    top = oracle.topk(oracle.indexer(inp["qI"], inp["w"], inp["kI"], np.arange(N)),
                      np.arange(N) + 1, 10)
    ptr, idx = oracle.selection(top, 5, np.arange(N))
    q = oracle._f64(inp["q"])
    ones = np.ones((N, 64))
    out, _ = oracle.sparse_attention(q, oracle._f64(inp["k"]), ones, ptr, idx, 0.125)
    assert np.max(np.abs(out - 1.0)) < 1e-12           # sum_s p_s = 1
    _, lse = oracle.sparse_attention(np.zeros_like(q), oracle._f64(inp["k"]), ones, ptr, idx, 0.125)
    n = np.diff(ptr)
    assert np.max(np.abs(lse - np.log(n)[:, None])) < 1e-12   # uniform logits


def test_attention_single_key_and_order_invariance():
    inp = gen_prefill(N=40, Hq=2, d=64, H_I=2, D_I=32, seed=8)
    q, k, v = (oracle._f64(inp[x]) for x in "qkv")
    out, _ = oracle.sparse_attention(q[:1], k, v, np.array([0, 1]), np.array([17]), 0.125)
    assert np.array_equal(out[0], np.stack([v[17], v[17]]))
    idx = np.array([3, 9, 12, 30, 31])
    a, _ = oracle.sparse_attention(q[31:32], k, v, np.array([0, 5]), idx, 0.125)
    b, _ = oracle.sparse_attention(q[31:32], k, v, np.array([0, 5]), idx[::-1].copy(), 0.125)
    assert np.max(np.abs(a - b)) < 1e-14


def test_decode_equals_last_prefill_row():
    L = 300
    dec = gen_decode(B=1, L=L, Hq=4, d=64, H_I=2, D_I=32, seed=9)
    pre = dict(q=np.repeat(dec["q"], 1, axis=0), k=dec["k"][0], v=dec["v"][0],
               qI=dec["qI"], w=dec["w"], kI=dec["kI"][0])
    rd = oracle.decode(dec, K=40, W=16)
    rp = oracle.prefill(dict(pre, q=np.concatenate([np.zeros((L - 1, 4, 64), np.uint16), dec["q"]]),
                             qI=np.concatenate([np.zeros((L - 1, 2, 32), np.uint16), dec["qI"]]),
                             w=np.concatenate([np.zeros((L - 1, 2), np.uint16), dec["w"]])),
                        K=40, W=16, rows=[L - 1])
    assert np.array_equal(rd["topk"], rp["topk"])
    assert np.max(np.abs(rd["out"] - rp["out"])) == 0.0


def test_paged_decode_equals_contiguous():
    lengths = [130, 64, 1, 200]
    cont = gen_decode(B=4, lengths=lengths, Hq=2, d=64, H_I=2, D_I=32, seed=4)
    paged = gen_decode(B=4, lengths=lengths, Hq=2, d=64, H_I=2, D_I=32, seed=4, paged=True)
    # rebuild the paged pools from the contiguous data through the table
    for name in ("k", "v", "kI"):
        pool = np.zeros_like(paged[name])
        for b, L in enumerate(lengths):
            for s in range(L):
                pool[paged["page_table"][b, s // 64], s % 64] = cont[name][b, s]
        paged[name] = pool
    a, b = oracle.decode(cont, K=16, W=8), oracle.decode(paged, K=16, W=8)
    assert np.array_equal(a["topk"], b["topk"]) and np.array_equal(a["out"], b["out"])


def test_bf16_rounding_of_inputs():
    x = np.array([1.0, 1.00390625, 1.005859375, -2.5, 3.0], dtype=np.float32)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: rounds to even (1.0);
    # 1 + 1.5 * 2^-8 rounds up to 1 + 2^-7.
    got = oracle._f64(bf16_bits(x))
    assert list(got) == [1.0, 1.0, 1.0078125, -2.5, 3.0]
