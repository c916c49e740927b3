"""GPU parity of the page-granular selection: whole kept blocks plus the
query's own block, with no fine selection.  It runs on the two-stage path with
a fine top-K that may keep every candidate (K = keep*block + block), so each
query attends to all tokens of its kept blocks, its own block up to itself
and its window.  Index sets must match the oracle bit for bit; outputs within
max-abs 2e-2 and mean-abs 2e-3 of the fp64 result."""

import numpy as np
import pytest
import torch

import oracle
from workloads import gen_prefill
from tests.gpu_helpers import assert_close_attention, dev, host_f64, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_top_b200 as m
    return m


@pytest.mark.parametrize("N,block,keep,W,rows", [
    (1000, 64, 4, 16, None),       # every row; short rows keep fewer than `keep` blocks
    (4096, 64, 16, 64, 300),       # sampled rows, up to 16 kept blocks of 64 + own block
])
def test_page_selection_matches_oracle(sa, N, block, keep, W, rows):
    from fine_grained_top_b200.pipeline import PrefillPlan
    inp = gen_prefill(N=N, Hq=16, d=128, H_I=4, D_I=64, seed=N + keep)
    K = keep * block + block
    plan = PrefillPlan(N, 16, 128, 4, 64, K, W, block=block, keep=keep)
    t = {n: dev(inp[n]) for n in ("q", "k", "v", "qI", "w", "kI")}
    plan.run(t["q"], t["k"], t["v"], t["qI"], t["w"], t["kI"])
    assert status(plan.dev_status) == 0
    r = np.arange(N) if rows is None else np.unique(np.r_[np.linspace(0, N - 1, rows).astype(int), 63, 64])
    pos, blocks = oracle.page_selection(r, inp["qI"][r], inp["w"][r], inp["kI"], block, keep)
    got = plan.topk.cpu().numpy()[r]
    assert np.array_equal(got, pos)
    # every kept position is a whole kept block or the own block: a page-granular set
    for i, t_ in enumerate(r):
        sel = got[i][got[i] >= 0]
        own = t_ // block
        full = sel[sel < own * block]
        assert len(full) % block == 0 and np.all(full.reshape(-1, block) % block == np.arange(block)), t_
        assert np.array_equal(sel[sel >= own * block], np.arange(own * block, t_ + 1)), t_
    ref = oracle.prefill(inp, K, W, rows=r, block=block, keep=keep)
    assert np.array_equal(ref["topk"], pos)
    assert_close_attention(host_f64(plan.out)[r], ref["out"], "out")
