"""sa_sparse_attn_decode_noalloc against the CPU fp64 oracle and the regular decode.

The allocation-free decode exists for callers that cannot allocate device
memory (a plugin in an engine that owns all of the GPU's memory and passes
only inputs and outputs; a loop where cudaMalloc / cudaFree must not run).
It keeps its split partials in a fixed array inside the library instead of a
caller workspace, and always runs the split-K kernels and their merge kernel.
This test calls it twice in a row through the C ABI -- on two different
problems, so the second call starts from the first call's leftovers in the
shared array.  Each result is checked against the oracle's decode on the same
inputs, within the attention tolerance used by every other GPU test, and
against the regular entry point's output.  It passes alone in a fresh process
and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import gen_decode
from tests.gpu_helpers import MAX_ABS, MEAN_ABS, dev, host_f64, status

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import fine_grained_top_b200 as m
    return m


def _one_call(sa, lengths, paged, K, W, seed):
    from fine_grained_top_b200.pipeline import DecodePlan
    B, Hq, d, H_I, D_I = len(lengths), 64, 128, 8, 64
    inp = gen_decode(B=B, lengths=lengths, Hq=Hq, d=d, H_I=H_I, D_I=D_I, paged=paged, seed=seed)
    x = {k: dev(inp[k]) for k in ("q", "k", "v", "qI", "w", "kI")}
    sl = dev(inp["lengths"])
    if paged:
        pt, mp, pp, s_max = dev(inp["page_table"]), inp["page_table"].shape[1], inp["k"].shape[0], 0
    else:
        pt, mp, pp, s_max = None, 0, 0, inp["k"].shape[1]
    plan = DecodePlan(B, Hq, d, H_I, D_I, K, W, S_max=s_max, paged=paged, max_pages=mp, pool_pages=pp)
    plan.run(x["q"], x["k"], x["v"], x["qI"], x["w"], x["kI"], sl, pt)     # existing entry points
    assert status(plan.dev_status) == 0
    out = torch.empty_like(plan.out)
    lse = torch.empty_like(plan.lse)
    ds = torch.zeros(1, dtype=torch.int32, device="cuda")
    sa.sa_sparse_attn_decode_noalloc(x["q"], x["k"], x["v"], pt, mp, pp, 64, s_max, sl, plan.topk, K, W, B,
                                     Hq, d, plan.scale, out, lse, ds)
    assert status(ds) == 0
    ref = oracle.decode(inp, K, W)
    assert np.array_equal(plan.topk.cpu().numpy(), ref["topk"])
    got = host_f64(out)
    assert np.all(np.isfinite(got))
    err = np.abs(got - ref["out"])
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert np.max(np.abs(host_f64(lse) - ref["lse"])) < 1e-3
    # and the regular entry point on the same selection
    err2 = np.abs(got - host_f64(plan.out))
    assert err2.max() <= MAX_ABS and err2.mean() <= MEAN_ABS, (err2.max(), err2.mean())


def test_noalloc_decode_matches_workspace_decode_twice(sa):
    # first call: 16 sequences on a paged cache (about 10.5 MB of partials)
    _one_call(sa, [16384, 262144, 70000, 5000, 1, 64, 65, 200000, 131072, 33333, 100000, 2048, 4097,
                   250000, 99, 180000], True, 2048, 512, seed=21)
    # second call: a different, smaller problem on a contiguous cache
    _one_call(sa, [131072, 3000, 777], False, 1024, 256, seed=22)


def test_noalloc_rejects_oversized_calls(sa):
    # B * splits * Hq * (d + 1) * 4 bytes beyond the fixed array: refused, nothing enqueued
    B = 64
    need = sa.sa_decode_workspace_bytes(B, 64, 128, 2048, 512)
    assert need > sa.SA_DECODE_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((B, 64, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((B, 16, 128), dtype=torch.bfloat16, device="cuda")
    sl = torch.full((B,), 16, dtype=torch.int32, device="cuda")
    top = torch.full((B, 2048), -1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(sa.SAError) as e:
        sa.sa_sparse_attn_decode_noalloc(q, kv, kv, None, 0, 0, 64, 16, sl, top, 2048, 512, B, 64, 128,
                                         0.1, out)
    assert e.value.status == sa.SA_ERR_WORKSPACE
