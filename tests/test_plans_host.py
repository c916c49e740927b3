"""Host logic of the step plans, on CPU (plans only allocate buffers and pick
entry points when they are built; nothing here launches a kernel):
attention-path dispatch, buffer shapes and the kernel count of a step."""

import pytest

from tests.conftest import ROOT  # noqa: F401  (puts the repo on sys.path)


@pytest.fixture(scope="module")
def pl():
    import __graft_entry__
    __graft_entry__.build()
    import fine_grained_top_b200 as sa
    from fine_grained_top_b200 import pipeline
    return sa, pipeline


def test_prefill_8k_takes_the_masked_tensor_core_attention(pl):
    sa, pipeline = pl
    p = pipeline.PrefillPlan(8192, 16, 128, 4, 64, 1024, 128, device="cpu")
    # 8192 * 16 query-head rows / 256 per CTA = 512 CTAs >= 148 SMs, and the
    # selection is dense enough: the bitmap workspace is allocated
    assert p.attn_ws_bytes == sa.sa_prefill_workspace_bytes(8192, 8192, 1024, 128, 16, 128) == 8192 * 256 * 4
    assert p.attn_ws is not None and p.attn_ws.numel() == p.attn_ws_bytes
    assert tuple(p.scores.shape) == (8192, 8192) and tuple(p.topk.shape) == (8192, 1024)
    assert p.launches() == 4                 # indexer, top-K, selection bitmap, masked attention
    assert p.index is sa.sa_indexer_scores


def test_small_prefill_takes_the_gathered_attention(pl):
    _, pipeline = pl
    p = pipeline.PrefillPlan(512, 4, 64, 2, 32, 64, 32, device="cpu")
    assert p.attn_ws is None and p.attn_ws_bytes == 0   # 8 CTAs of the masked kernel would idle 140 SMs
    assert p.launches() == 3
    assert p.ld % 4 == 0 and p.ld >= 512


def test_two_stage_and_page_granular_plans(pl):
    _, pipeline = pl
    p = pipeline.PrefillPlan(4096, 16, 128, 4, 64, 512, 64, block=64, keep=16, device="cpu")
    assert p.nb == 64 and tuple(p.blocks.shape) == (4096, 16)
    assert p.ld_cand == 16 * 64 + 64 and tuple(p.fine.shape) == (4096, p.ld_cand)
    assert p.launches() == 9 + 2        # 9 selection kernels (no candidate map), bitmap, masked attention
    names = [n for n, _ in p.stages({k: None for k in ("q", "k", "v", "qI", "w", "kI")})]
    assert names == ["pool", "block_counts", "coarse_indexer", "coarse_topk", "fine_indexer", "fine_topk",
                     "attention"]
    # page-granular: the fine top-K may keep every candidate
    q = pipeline.PrefillPlan(4096, 16, 128, 4, 64, 16 * 64 + 64, 64, block=64, keep=16, device="cpu")
    assert tuple(q.topk.shape) == (4096, q.ld_cand)
    with pytest.raises(ValueError):
        pipeline.PrefillPlan(4096, 16, 128, 4, 64, 512, 64, block=64, keep=16, index_fp8=True, device="cpu")


def test_row_blocked_plan_counts_its_launches(pl):
    _, pipeline = pl
    p = pipeline.PrefillPlan(8192, 16, 128, 4, 64, 1024, 128, row_blocks=4, device="cpu")
    assert p.launches() == 2 * 4 + 2
    names = [n for n, _ in p.stages({k: None for k in ("q", "k", "v", "qI", "w", "kI")})]
    assert names == ["indexer", "topk"] * 4 + ["attention"]


def test_decode_plans(pl):
    sa, pipeline = pl
    d = pipeline.DecodePlan(8, 64, 128, 8, 64, 2048, 512, S_max=131072, device="cpu")
    assert d.ws_bytes == sa.sa_decode_workspace_bytes(8, 64, 128, 2048, 512) > 0
    # indexer and top-K apart by default; cluster decode: no merge kernel
    assert not d.fused and d.launches() == 3 and d.index is sa.sa_indexer_scores
    fd = pipeline.DecodePlan(8, 64, 128, 8, 64, 2048, 512, S_max=131072, fused=True, device="cpu")
    assert fd.fused and fd.launches() == 2 and fd.scores is None
    names = [n for n, _ in fd.stages({k: None for k in ("q", "k", "v", "qI", "w", "kI", "lengths")})]
    assert names == ["indexer_topk", "attention"]
    # K + W beyond 16 CTAs x 1024 keys takes split-K + merge
    big = pipeline.DecodePlan(2, 64, 128, 8, 64, 20000, 512, S_max=65536, device="cpu")
    assert big.launches() == 4
    # shapes the fused kernel does not take
    for H_I, D_I, S in ((16, 64, 4096), (8, 32, 4096), (8, 64, 524288)):
        with pytest.raises(ValueError):
            pipeline.DecodePlan(2, 64, 128, H_I, D_I, 2048, 512, S_max=S, fused=True, device="cpu")
    assert d.ld >= 131072 and d.ld % 4 == 0
    f = pipeline.DecodePlan(16, 64, 128, 8, 64, 2048, 512, S_max=0, paged=True, max_pages=4096,
                            pool_pages=40000, index_fp8=True, device="cpu")
    assert f.S == 4096 * 64 and f.index is sa.sa_indexer_scores_fp8
    names = [n for n, _ in f.stages({k: None for k in ("q", "k", "v", "qI", "w", "kI", "lengths")})]
    assert names == ["indexer", "topk", "attention"]
