"""The multi-rank partitions of the path (fine_grained_top_b200.shard) on CPU.

Two `gloo` ranks run the partitioned step's host logic -- row-chunk bounds,
key shards, the one all-gather of k, v and kI, each rank's rows as the last
rows of a shorter sequence -- with the CPU oracle standing in for the CUDA
plan, and the partitioned results must equal the unpartitioned oracle's on
every row (index sets bit for bit, outputs exactly: both sides are the same
fp64 code on the same rows).  The decode split deals whole sequences.  No GPU
is needed; the CUDA plans behind the same partition are unmeasured on more
than one GPU.
"""

import os
import socket

import numpy as np
import pytest

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# ---------------------------------------------------------------- host logic
@pytest.mark.parametrize("N,world", [(1, 2), (7, 3), (700, 2), (8192, 8), (65536, 8), (1000, 4)])
@pytest.mark.parametrize("two_stage", [False, True])
def test_chunk_bounds_cover_and_balance(N, world, two_stage):
    from fine_grained_top_b200.shard import causal_chunk_bounds, prefill_row_cost
    kw = dict(block=64, keep=64) if two_stage else {}
    cost = prefill_row_cost(N, 2048, 512, 16, 128, 4, 64, **kw)
    b = causal_chunk_bounds(cost, world)
    assert b[0] == 0 and b[-1] == N and len(b) == world + 1
    assert all(b[i] <= b[i + 1] for i in range(world))
    per = [cost[b[i]:b[i + 1]].sum() for i in range(world)]
    # each chunk is within one row's cost of an equal share
    assert max(per) <= cost.sum() / world + cost.max() + 1e-6


def test_row_cost_counts_the_scored_keys():
    from fine_grained_top_b200.shard import prefill_row_cost
    # single stage: row t scores t + 1 keys and attends to min(t + 1, K + W)
    c = prefill_row_cost(10, 3, 2, 1, 1, 1, 1)
    assert np.allclose(c, 2 * np.arange(1, 11) + 4 * np.minimum(np.arange(1, 11), 5))
    # two stage, block 4, keep 2: row 9 scores 2 coarse blocks, 2 kept blocks of 4 and its own 2 tokens
    c2 = prefill_row_cost(10, 100, 0, 1, 1, 1, 1, block=4, keep=2)
    assert c2[9] == 2 * (2 + 2 * 4 + 2) + 4 * 10


def test_decode_assignment_deals_every_sequence_once():
    from fine_grained_top_b200.shard import decode_assignment
    rng = np.random.default_rng(0)
    lengths = rng.integers(16384, 262145, size=16)
    for world in (1, 2, 3, 8, 16, 20):
        owned = decode_assignment(lengths, world)
        flat = sorted(b for o in owned for b in o)
        assert flat == list(range(16))
        loads = [int(lengths[o].sum()) if o else 0 for o in owned]
        assert max(loads) <= lengths.sum() / world + lengths.max()


def test_key_shards_cover_the_sequence():
    from fine_grained_top_b200.shard import key_shard_bounds
    for N, world in ((10, 3), (65536, 8), (5, 8)):
        b = key_shard_bounds(N, world)
        assert b[0] == 0 and b[-1] == N and all(b[i] <= b[i + 1] for i in range(world))


# ---------------------------------------------------------------- gloo ranks
class OraclePlan:
    """The plan interface (run(q, k, v, qI, w, kI) for T queries at the last T
    of S keys) computed by the CPU oracle; bf16 tensors travel as int16."""

    def __init__(self, T, S, K, W, block, keep):
        self.T, self.S, self.K, self.W, self.block, self.keep = T, S, K, W, block, keep

    def run(self, q, k, v, qI, w, kI):
        import oracle
        bits = lambda t: t.numpy().view(np.uint16)
        T, S = self.T, self.S
        def rows_at_end(x):
            full = np.zeros((S,) + x.shape[1:], dtype=np.uint16)
            full[S - T:] = x
            return full
        inp = {"q": rows_at_end(bits(q)), "qI": rows_at_end(bits(qI)), "w": rows_at_end(bits(w)),
               "k": bits(k), "v": bits(v), "kI": bits(kI)}
        self.res = oracle.prefill(inp, self.K, self.W, rows=np.arange(S - T, S), block=self.block, keep=self.keep)
        return self.res


def _prefill_rank(rank, world, port, out_dir, case):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from fine_grained_top_b200.shard import ShardedPrefill, key_shard_bounds
    from workloads import gen_prefill
    N, Hq, d, H_I, D_I, K, W, block, keep = case
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), ORACLE_THREADS="2")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = gen_prefill(N=N, Hq=Hq, d=d, H_I=H_I, D_I=D_I, seed=5)
        t16 = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16))
        sp = ShardedPrefill(N, Hq, d, H_I, D_I, K, W, rank, world, block=block, keep=keep, device="cpu",
                            make_plan=lambda T, S: OraclePlan(T, S, K, W, block, keep))
        kb = key_shard_bounds(N, world)
        ks = slice(kb[rank], kb[rank + 1])
        rs = slice(sp.t0, sp.t1)
        k_full, v_full, kI_full = sp.gather_keys(t16(inp["k"][ks]), t16(inp["v"][ks]), t16(inp["kI"][ks]))
        gathered_ok = (np.array_equal(k_full.numpy().view(np.uint16), inp["k"][:sp.t1]) and
                       np.array_equal(v_full.numpy().view(np.uint16), inp["v"][:sp.t1]) and
                       np.array_equal(kI_full.numpy().view(np.uint16), inp["kI"][:sp.t1]))
        res = sp.run(t16(inp["q"][rs]), t16(inp["qI"][rs]), t16(inp["w"][rs]),
                     t16(inp["k"][ks]), t16(inp["v"][ks]), t16(inp["kI"][ks]))
    finally:
        dist.destroy_process_group()
    if res is None:
        res = {"topk": np.zeros((0, K), np.int64), "out": np.zeros((0, Hq, d)), "lse": np.zeros((0, Hq))}
    np.savez(os.path.join(out_dir, "rank%d.npz" % rank), t0=sp.t0, t1=sp.t1, gathered_ok=gathered_ok,
             topk=res["topk"], out=res["out"], lse=res["lse"])


@pytest.mark.parametrize("case", [
    (700, 4, 64, 2, 32, 64, 16, None, None),       # single-stage selection
    (1000, 4, 64, 2, 32, 100, 16, 64, 4),           # two-stage selection
])
def test_two_gloo_ranks_prefill_partition_equals_whole(tmp_path, case):
    import torch.multiprocessing as mp
    import oracle
    from workloads import gen_prefill
    world = 2
    mp.start_processes(_prefill_rank, args=(world, _free_port(), str(tmp_path), case), nprocs=world,
                       start_method="spawn", join=True)
    parts = [np.load(tmp_path / ("rank%d.npz" % r)) for r in range(world)]
    N, Hq, d, H_I, D_I, K, W, block, keep = case
    assert [int(p["t0"]) for p in parts] == [0, int(parts[0]["t1"])] and int(parts[1]["t1"]) == N
    assert 0 < int(parts[0]["t1"]) < N   # both ranks own rows
    assert all(bool(p["gathered_ok"]) for p in parts)
    whole = oracle.prefill(gen_prefill(N=N, Hq=Hq, d=d, H_I=H_I, D_I=D_I, seed=5), K, W, block=block, keep=keep)
    assert np.array_equal(np.concatenate([p["topk"] for p in parts]), whole["topk"])
    assert np.array_equal(np.concatenate([p["out"] for p in parts]), whole["out"])
    assert np.array_equal(np.concatenate([p["lse"] for p in parts]), whole["lse"])


def _decode_rank(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    from fine_grained_top_b200.shard import decode_assignment
    from workloads import gen_decode
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), ORACLE_THREADS="2")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = gen_decode(B=5, lengths=[3000, 70, 9000, 1, 4097], Hq=8, d=64, H_I=2, D_I=32, paged=True, seed=4)
        mine = decode_assignment(inp["lengths"], world)[rank]
        res = oracle.decode(inp, 64, 16, seqs=mine)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    np.savez(os.path.join(out_dir, "rank%d.npz" % rank), seqs=np.array(mine, np.int64), topk=res["topk"],
             out=res["out"], lse=res["lse"])


def test_two_gloo_ranks_decode_split_equals_whole(tmp_path):
    import torch.multiprocessing as mp
    import oracle
    from workloads import gen_decode
    world = 2
    mp.start_processes(_decode_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    parts = [np.load(tmp_path / ("rank%d.npz" % r)) for r in range(world)]
    seqs = np.concatenate([p["seqs"] for p in parts])
    assert sorted(seqs.tolist()) == list(range(5)) and all(len(p["seqs"]) for p in parts)
    whole = oracle.decode(gen_decode(B=5, lengths=[3000, 70, 9000, 1, 4097], Hq=8, d=64, H_I=2, D_I=32, paged=True,
                                     seed=4), 64, 16)
    for key in ("topk", "out", "lse"):
        got = np.concatenate([p[key] for p in parts])
        assert np.array_equal(got, whole[key][seqs])


# ---------------------------------------------------------------- collecting results on every rank
def _collect_rank(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import oracle
    from fine_grained_top_b200.shard import ShardedDecode, ShardedPrefill, gather_chunks
    from workloads import gen_decode, gen_prefill
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), ORACLE_THREADS="2")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # prefill: each rank's rows, then the whole sequence's results on every rank
        N, Hq, d, H_I, D_I, K, W = 600, 4, 64, 2, 32, 64, 16
        inp = gen_prefill(N=N, Hq=Hq, d=d, H_I=H_I, D_I=D_I, seed=9)
        sp = ShardedPrefill(N, Hq, d, H_I, D_I, K, W, rank, world, device="cpu", make_plan=lambda T, S: None)
        rows = np.arange(sp.t0, sp.t1)
        mine = oracle.prefill(inp, K, W, rows=rows) if len(rows) else \
            {"topk": np.zeros((0, K), np.int64), "out": np.zeros((0, Hq, d)), "lse": np.zeros((0, Hq))}
        full_p = {k: sp.collect(torch.from_numpy(np.ascontiguousarray(mine[k]))).numpy()
                  for k in ("topk", "out", "lse")}
        # decode: whole sequences per rank, results back in batch order on every rank
        lengths = [3000, 70, 9000, 1, 4097, 640]
        dinp = gen_decode(B=len(lengths), lengths=lengths, Hq=8, d=64, H_I=2, D_I=32, paged=True, seed=4)
        sd = ShardedDecode(lengths, rank, world)
        dres = oracle.decode(dinp, 64, 16, seqs=sd.owned)
        full_d = {k: sd.collect(torch.from_numpy(np.ascontiguousarray(dres[k]))).numpy() for k in ("topk", "out", "lse")}
        picked = sd.select(np.asarray(lengths))
        # an empty chunk on one rank, and a dtype other than the defaults
        local = (torch.arange(3 * rank, dtype=torch.int16).reshape(rank, 3) if rank
                 else torch.zeros((0, 3), dtype=torch.int16))
        ragged = gather_chunks(local, [0, 0] + [world - 1], None).numpy() if world == 2 else None
        dist.barrier()
    finally:
        dist.destroy_process_group()
    np.savez(os.path.join(out_dir, "c%d.npz" % rank), owned=np.array(sd.owned, np.int64), picked=picked,
             ragged=ragged, **{"p_" + k: v for k, v in full_p.items()}, **{"d_" + k: v for k, v in full_d.items()})


def test_two_gloo_ranks_collect_full_results():
    import tempfile
    import torch.multiprocessing as mp
    import oracle
    from workloads import gen_decode, gen_prefill
    world = 2
    with tempfile.TemporaryDirectory() as tmp:
        mp.start_processes(_collect_rank, args=(world, _free_port(), tmp), nprocs=world, start_method="spawn",
                           join=True)
        parts = [dict(np.load(os.path.join(tmp, "c%d.npz" % r), allow_pickle=True)) for r in range(world)]
    whole = oracle.prefill(gen_prefill(N=600, Hq=4, d=64, H_I=2, D_I=32, seed=9), 64, 16)
    lengths = [3000, 70, 9000, 1, 4097, 640]
    dwhole = oracle.decode(gen_decode(B=6, lengths=lengths, Hq=8, d=64, H_I=2, D_I=32, paged=True, seed=4), 64, 16)
    for p in parts:   # every rank holds the whole result, in query / batch order
        for k in ("topk", "out", "lse"):
            assert np.array_equal(p["p_" + k], whole[k]), k
            assert np.array_equal(p["d_" + k], dwhole[k]), k
        assert np.array_equal(p["picked"], np.asarray(lengths)[p["owned"]])
        assert np.array_equal(p["ragged"], np.arange(3, dtype=np.int16).reshape(1, 3))   # rank 0 sent no rows
    assert sorted(np.concatenate([p["owned"] for p in parts]).tolist()) == list(range(6))
